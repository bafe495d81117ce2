// Attention with summed weights for chunks of a few tokens (decode-sized:
// G * S <= 16 query rows per KV head), split over the keys.
//
// "Learning how to Forget: Fine-tuning for Long-Context Sparse Attention",
// FAQ answer 3 (SDPA that also returns the summed attention weights); §1 ¶1
// (attention over a fixed-size cache), §1 ¶3 (GQA).
//
// With so few rows the step is bound by reading the cache once, not by
// arithmetic, so this kernel uses plain FMA dot products: one thread-block
// cluster of kc CTAs per (b, KV head), CTA `rank` taking a contiguous run of
// the visible keys (the valid cache slots, then the chunk's keys).  A warp
// takes a key at a time: lane l holds D/32 consecutive elements of the row
// (one coalesced load), the dot products with all rows are summed across the
// warp, and the scores stay in shared memory for the second sweep, so K is
// read once.
//   sweep 1: each row's running (max, sum), per warp, then per CTA, then over
//            the cluster in rank order through distributed shared memory, so
//            every CTA holds the same log-sum-exp;
//   sweep 2: p = 2^(s - lse), the key's column sum over all rows (added to
//            the KV head's accumulator row: each key belongs to one CTA),
//            O += p v per warp; the warps' O are added in warp order, and rank
//            q adds the CTAs' O of rows r = q (mod kc) in rank order.
#include "h2o_internal.cuh"

namespace h2o {
namespace {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecMaxCluster = 16;

__device__ __forceinline__ void from_f(float x, float* p) { *p = x; }
__device__ __forceinline__ void from_f(float x, __nv_bfloat16* p) { *p = __float2bfloat16_rn(x); }

__device__ __forceinline__ uint32_t dec_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void dec_cluster_sync() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t dec_map(const void* p, uint32_t rank) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
__device__ __forceinline__ float dec_ld(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2f(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// E consecutive elements of a row into floats, one vector load
template <typename T, int E>
__device__ __forceinline__ void load_row(const T* src, float (&x)[E]) {
  if constexpr (sizeof(T) == 2 && E == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(src);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
  } else if constexpr (sizeof(T) == 2 && E == 2) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(src));
    x[0] = a.x; x[1] = a.y;
  } else if constexpr (sizeof(T) == 4 && E == 4) {
    const float4 a = *reinterpret_cast<const float4*>(src);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  } else {
    const float2 a = *reinterpret_cast<const float2*>(src);
    x[0] = a.x; x[1] = a.y;
  }
}

// Lane l of 32 partial sums v[0..31] ends with the sum over the warp of
// v[l] (31 shuffles: each step keeps half of the values and adds the other
// lane's copy of them).
__device__ __forceinline__ float transpose_reduce(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const bool hi = lane & o;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = hi ? v[i] : v[i + o];
      const float keep = hi ? v[i + o] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return v[0];
}

// Keys are taken in batches of kKB per warp (their rows loaded together, so
// that 16 row loads per lane are in flight); within a batch, rounds of 32 / RM
// keys x RM rows = 32 dot products are reduced at once: lane l then holds the
// score of key u = l / RM, row r = l % RM of the round.
constexpr int kKB = 16;

template <typename T, int D, int RM>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(const DecodeArgs a) {
  constexpr int E = D / 32;                       // row elements per lane
  constexpr int KR = 32 / RM;                     // keys per round
  constexpr int NR = kKB / KR;                    // rounds per batch
  static_assert(kKB % KR == 0, "batch of whole rounds");
  extern __shared__ __align__(16) float sbuf[];   // [per][RM] scores, base 2
  __shared__ float ml_w[kDecWarps][RM][2];        // warps' (max, sum)
  __shared__ float ml_c[RM][2];                   // this CTA's (max, sum): read by the cluster
  __shared__ float lse[RM];
  __shared__ float o_c[RM][D];                    // this CTA's O: read by the cluster
  __shared__ float o_w[kDecWarps][D];             // scratch for the warp reduction of one row

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = dec_rank();
  const int kc = a.kc;
  const int bh = blockIdx.x / kc;
  const int b = bh / a.Hkv, h = bh - b * a.Hkv;
  const int64_t S = a.S, nv = a.n_valid, M = a.M;
  const int R = a.G * (int)S;                     // rows: (local head g, chunk row i), r = g * S + i
  const int64_t keys = nv + S;
  const int64_t per = a.per;
  const int64_t k0 = (int64_t)rank * per, k1 = k0 + per < keys ? k0 + per : keys;
  const T* q = static_cast<const T*>(a.q);
  const T* kb = static_cast<const T*>(a.k) + (int64_t)bh * S * D;
  const T* vb = static_cast<const T*>(a.v) + (int64_t)bh * S * D;
  const T* kcb = static_cast<const T*>(a.kcache) + (int64_t)bh * M * D;
  const T* vcb = static_cast<const T*>(a.vcache) + (int64_t)bh * M * D;
  unsigned long long* acc = a.colacc + (int64_t)bh * a.acc_stride;   // the KV head's accumulator row
  const int my_r = lane % RM, my_u = lane / RM;   // lane's (row, key in round) after a reduction
  const int my_i = my_r < R ? my_r % (int)S : -1; // its chunk row (causal limit); -1: no such row

  // the previous kernel of the stream may still be writing the cache
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // this lane's elements of every row, scaled by log2(e) / sqrt(d)
  float qr[RM][E];
#pragma unroll
  for (int r = 0; r < RM; ++r) {
    if (r < R) {
      const int g = r / (int)S, i = r - g * (int)S;
      load_row<T, E>(q + (((int64_t)b * a.Hq + h * a.G + g) * S + i) * D + lane * E, qr[r]);
#pragma unroll
      for (int e = 0; e < E; ++e) qr[r][e] *= a.scale_log2;
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) qr[r][e] = 0.f;
    }
  }
  // a batch's rows, loaded without branches (a key past the CTA's run reloads
  // its last key, whose score and weight are then ignored), so that all the
  // batch's loads are in flight together
  auto load_batch = [&](const T* cache_rows, const T* chunk_rows, int64_t j0, float (&x)[kKB][E]) {
    const T* src[kKB];
#pragma unroll
    for (int u = 0; u < kKB; ++u) {
      const int64_t j = j0 + u < k1 ? j0 + u : k1 - 1;
      src[u] = (j < nv ? cache_rows + j * D : chunk_rows + (j - nv) * D) + lane * E;
    }
#pragma unroll
    for (int u = 0; u < kKB; ++u) load_row<T, E>(src[u], x[u]);
  };

  // ---- sweep 1: scores to shared memory; each lane keeps a running (max, sum)
  // of its row over the keys it is handed
  float m = -INFINITY, l = 0.f;
  for (int64_t j0 = k0 + (int64_t)warp * kKB; j0 < k1; j0 += (int64_t)kDecWarps * kKB) {
    float kx[kKB][E];
    load_batch(kcb, kb, j0, kx);
#pragma unroll
    for (int rd = 0; rd < NR; ++rd) {
      float v[32];
#pragma unroll
      for (int u = 0; u < KR; ++u)
#pragma unroll
        for (int r = 0; r < RM; ++r) {
          float d = 0.f;
#pragma unroll
          for (int e = 0; e < E; ++e) d = fmaf(qr[r][e], kx[rd * KR + u][e], d);
          v[u * RM + r] = d;
        }
      const float sc = transpose_reduce(v);
      const int64_t j = j0 + rd * KR + my_u;
      if (j < k1) {
        const bool vis = my_i >= 0 && (j < nv || j - nv <= my_i);
        const float x = vis ? sc : -INFINITY;
        sbuf[(j - k0) * RM + my_r] = x;
        if (x > m) {
          l = (m == -INFINITY ? 0.f : l * ex2f(m - x)) + 1.f;
          m = x;
        } else if (vis) {
          l += ex2f(x - m);
        }
      }
    }
  }
  // the warp's (max, sum) of each row: lanes r, r + RM, ... hold its parts
#pragma unroll
  for (int o = RM; o < 32; o <<= 1) {
    const float mo = __shfl_xor_sync(0xffffffffu, m, o), lo = __shfl_xor_sync(0xffffffffu, l, o);
    const float mx = fmaxf(m, mo);
    const float nl = (l > 0.f ? l * ex2f(m - mx) : 0.f) + (lo > 0.f ? lo * ex2f(mo - mx) : 0.f);
    m = mx;
    l = nl;
  }
  if (lane < RM) {
    ml_w[warp][lane][0] = m;
    ml_w[warp][lane][1] = l;
  }
  __syncthreads();
  if (tid < RM) {   // the CTA's (max, sum) of row tid, warps in order
    float mx = -INFINITY;
    for (int w = 0; w < kDecWarps; ++w)
      if (ml_w[w][tid][1] > 0.f) mx = fmaxf(mx, ml_w[w][tid][0]);
    float sm = 0.f;
    for (int w = 0; w < kDecWarps; ++w)
      if (ml_w[w][tid][1] > 0.f) sm += ml_w[w][tid][1] * ex2f(ml_w[w][tid][0] - mx);
    ml_c[tid][0] = mx;
    ml_c[tid][1] = sm;
  }
  dec_cluster_sync();   // every CTA's (max, sum) is in its shared memory
  if (tid < RM) {       // the row's log-sum-exp over the cluster, ranks in order
    float mx = -INFINITY;
    for (int q2 = 0; q2 < kc; ++q2) {
      const float mq = dec_ld(dec_map(&ml_c[tid][0], (uint32_t)q2));
      const float lq = dec_ld(dec_map(&ml_c[tid][1], (uint32_t)q2));
      if (lq > 0.f) mx = fmaxf(mx, mq);
    }
    float sm = 0.f;
    for (int q2 = 0; q2 < kc; ++q2) {
      const float mq = dec_ld(dec_map(&ml_c[tid][0], (uint32_t)q2));
      const float lq = dec_ld(dec_map(&ml_c[tid][1], (uint32_t)q2));
      if (lq > 0.f) sm += lq * ex2f(mq - mx);
    }
    lse[tid] = sm > 0.f ? mx + lg2f(sm) : INFINITY;   // +inf: the row sees nothing
  }
  __syncthreads();

  // ---- sweep 2: p, column sums, O += p v (lane holds E elements of every row)
  const float my_lse = lse[my_r];
  float oa[RM][E];
#pragma unroll
  for (int r = 0; r < RM; ++r)
#pragma unroll
    for (int e = 0; e < E; ++e) oa[r][e] = 0.f;
  for (int64_t j0 = k0 + (int64_t)warp * kKB; j0 < k1; j0 += (int64_t)kDecWarps * kKB) {
    float vx[kKB][E];
    load_batch(vcb, vb, j0, vx);
#pragma unroll
    for (int rd = 0; rd < NR; ++rd) {
      const int64_t j = j0 + rd * KR + my_u;
      const float p = j < k1 ? ex2f(sbuf[(j - k0) * RM + my_r] - my_lse) : 0.f;   // -inf -> 0
      // the key's column sum over its RM rows (lanes u * RM .. u * RM + RM - 1)
      float cs = p;
#pragma unroll
      for (int o = 1; o < RM; o <<= 1) cs += __shfl_xor_sync(0xffffffffu, cs, o);
      if (my_r == 0 && j < k1) colsum_add(acc + (j < nv ? j : M + (j - nv)), cs, a.fx_scale);
#pragma unroll
      for (int u = 0; u < KR; ++u)
#pragma unroll
        for (int r = 0; r < RM; ++r) {
          const float pr = __shfl_sync(0xffffffffu, p, u * RM + r);
#pragma unroll
          for (int e = 0; e < E; ++e) oa[r][e] = fmaf(pr, vx[rd * KR + u][e], oa[r][e]);
        }
    }
  }
  // the CTA's O: warps added in warp order, one row at a time (the row index
  // is a compile-time constant of the unrolled loop: register arrays stay in registers)
#pragma unroll
  for (int r = 0; r < RM; ++r) {
#pragma unroll
    for (int e = 0; e < E; ++e) o_w[warp][lane * E + e] = oa[r][e];
    __syncthreads();
    for (int d = tid; d < D; d += kDecThreads) {
      float acc = 0.f;
      for (int w = 0; w < kDecWarps; ++w) acc += o_w[w][d];
      o_c[r][d] = acc;
    }
    __syncthreads();
  }
  dec_cluster_sync();   // every CTA's O is in its shared memory
  // rank q writes rows r = q, q + kc, ...: the CTAs' O added in rank order
  T* out = static_cast<T*>(a.out);
  if (out != nullptr) {
    for (int idx = tid; idx < RM * D; idx += kDecThreads) {
      const int r = idx / D, d = idx - r * D;
      if (r >= R || r % kc != (int)rank) continue;
      float acc = 0.f;
      for (int q2 = 0; q2 < kc; ++q2) acc += dec_ld(dec_map(&o_c[r][d], (uint32_t)q2));
      const int g = r / (int)S, i = r - g * (int)S;
      from_f(acc, out + (((int64_t)b * a.Hq + h * a.G + g) * S + i) * D + d);
    }
  }
  dec_cluster_sync();   // no CTA leaves while another reads its shared memory
}

template <typename T, int D, int RM>
cudaError_t launch_dec(const DecodeArgs& a, int BH, bool pdl, cudaStream_t st) {
  const size_t smem = (size_t)a.per * RM * sizeof(float);
  auto kern = decode_kernel<T, D, RM>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(BH * a.kc));
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = (unsigned)a.kc;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <typename T, int D>
cudaError_t launch_dec_rows(const DecodeArgs& a, int BH, bool pdl, cudaStream_t st) {
  return a.G * a.S <= 4 ? launch_dec<T, D, 4>(a, BH, pdl, st) : launch_dec<T, D, 16>(a, BH, pdl, st);
}

}  // namespace

// G * S <= 16 rows, and the scores of a CTA's keys fit its 160 KB with a
// portable cluster of 8 CTAs (16-row chunks up to 20480 keys, 4-row ones up to
// 81920); longer caches take the tensor-core path.
bool decode_supported(int G, int64_t S, int64_t keys) {
  if (S < 1 || G * S > 16) return false;
  const int RM = G * S <= 4 ? 4 : 16;
  return (keys + 7) / 8 * RM * 4 <= 160 * 1024;
}

// Keys per CTA and cluster size: at least 64 keys a CTA, scores within 160 KB
// of shared memory, and every (b, KV head) cluster in one wave if possible.
cudaError_t launch_decode(DecodeArgs a, int dtype, int BH, bool pdl, cudaStream_t st) {
  if (!decode_supported(a.G, a.S, a.n_valid + a.S) || (a.d != 64 && a.d != 128) || BH < 1) return cudaErrorInvalidValue;
  const int RM = a.G * a.S <= 4 ? 4 : 16;
  const int64_t keys = a.n_valid + a.S;
  int kc = 1;
  while (kc < kDecMaxCluster && keys / (2 * kc) >= 64) kc *= 2;
  while (kc < kDecMaxCluster && (keys + kc - 1) / kc * RM * 4 > 160 * 1024) kc *= 2;
  // fewer CTAs per cluster while the clusters would need more than one wave
  int sm = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sm, cudaDevAttrMultiProcessorCount, dev);
  while (kc > 1 && (int64_t)BH * kc > sm && (keys + kc / 2 - 1) / (kc / 2) * RM * 4 <= 160 * 1024) kc /= 2;
  if (kc > 8) kc = 8;   // portable cluster size: a 16-CTA cluster needs 16 free SMs of one GPC
  a.per = (keys + kc - 1) / kc;
  if (a.per * RM * 4 > 160 * 1024) return cudaErrorInvalidValue;
  a.kc = kc;
  if (dtype == kF32)
    return a.d == 64 ? launch_dec_rows<float, 64>(a, BH, pdl, st) : launch_dec_rows<float, 128>(a, BH, pdl, st);
  return a.d == 64 ? launch_dec_rows<__nv_bfloat16, 64>(a, BH, pdl, st)
                   : launch_dec_rows<__nv_bfloat16, 128>(a, BH, pdl, st);
}

}  // namespace h2o
