// Tensor-core (tcgen05 / TMEM / TMA) attention with summed attention weights,
// bf16 inputs, head dimension 128.
//
// "Learning how to Forget: Fine-tuning for Long-Context Sparse Attention":
// Abstract (H2O with a dedicated SDPA kernel), FAQ answer 3 (the SDPA kernel
// also returns the summed attention weights), §1 ¶1 (attention over a
// fixed-size cache), §1 ¶3 (GQA).
//
// One CTA owns 128 query rows of one query head (a row tile) and walks the
// keys it can see -- the valid cache slots, then the chunk's keys up to its
// causal limit -- in tiles of 128, twice:
//   sweep 1  S = Q K^T          (M = 128 queries, N = 128 keys)  -> row max and
//            sum of exp, i.e. each row's log-sum-exp;
//   sweep 2  S^T = K Q^T        (M = 128 keys, N = 128 queries), so each
//            softmax thread owns one key: it forms the exact probabilities
//            p = exp(s - lse) of its key for the 128 queries, sums them (its
//            column sum: no cross-thread reduction), and writes them to shared
//            memory as P^T; then O += P V (M = 128 queries, N = 128 = d) with P
//            read MN-major.
// Exact probabilities mean O needs no rescaling.  Each CTA writes one partial
// row of column sums (per key) that a fixed-order reduction adds up.
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 allocates TMEM
// and issues the MMAs (one thread), warps 2-5 (128 threads, thread = TMEM lane)
// do the softmax and the epilogue.  TMEM: two 128-column S buffers and a
// 128-column O accumulator.  Every mbarrier wait is bounded; a wait that runs
// out sets the kErrTimeout bit of the device error word and all roles exit.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <mutex>

#include "h2o_internal.cuh"
#include "sm100.cuh"

namespace h2o {
namespace {

using namespace sm100;

constexpr int BM = kUmmaRowTile;   // query rows per CTA
constexpr int BN = 128;            // keys per tile
constexpr int D = 128;             // head dimension
constexpr int NS = 2;              // K/V stages
constexpr int kThreads = 192;
constexpr uint32_t kAtom = BM * 64 * 2;          // one [128 x 64] bf16 box: 16 KB
constexpr uint32_t kTile = 2 * kAtom;            // [128 x 128] bf16: 32 KB
constexpr uint32_t kStage = 2 * kTile;           // K and V: 64 KB
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffKV = kOffQ + kTile;
constexpr uint32_t kOffP = kOffKV + NS * kStage;
constexpr uint32_t kOffLse = kOffP + kTile;
constexpr uint32_t kOffBar = kOffLse + BM * 4;
constexpr int kNumBars = 16;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemUsed = kOffMisc + 16;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;    // slack for 1024-byte alignment
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
constexpr uint64_t kWaitLimitNs = 1000000000ull;     // 1 s per wait

// barrier indices
enum { B_Q = 0, B_KV_FULL = 1, B_KV_EMPTY = B_KV_FULL + NS, B_S_FULL = B_KV_EMPTY + NS,
       B_S_EMPTY = B_S_FULL + 2, B_P_FULL = B_S_EMPTY + 2, B_P_EMPTY = B_P_FULL + 1,
       B_O_FULL = B_P_EMPTY + 1, B_DRAIN = B_O_FULL + 1 };
static_assert(B_DRAIN < kNumBars, "barrier count");

struct Params {
  float* partials;
  int* err;
  void* out;
  int B, Hq, Hkv, G, n_rt;
  int64_t S, M, n_valid;
  float scale_log2;   // (1/sqrt(d)) * log2(e)
};

__global__ void __launch_bounds__(kThreads, 1)
attn_umma_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kc,
                 const __grid_constant__ CUtensorMap tm_vc, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  float* lse2 = reinterpret_cast<float*>(sbase + kOffLse);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + kOffMisc + 4);
  auto bar = [&](int i) { return base + kOffBar + 8u * (uint32_t)i; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work unit: (b, h) major, then row tiles from the last (heaviest) one
  const int per_bh = p.G * p.n_rt;
  const int bh = blockIdx.x / per_bh;
  const int k_in = blockIdx.x - bh * per_bh;
  const int rt = p.n_rt - 1 - k_in / p.G;
  const int gl = k_in % p.G;
  const int b = bh / p.Hkv, h = bh - b * p.Hkv;
  const int g = h * p.G + gl;
  const int64_t i0 = (int64_t)rt * BM;
  const int nct = (int)((p.n_valid + BN - 1) / BN);        // cache tiles
  const int64_t chunk_hi = (i0 + BM < p.S) ? i0 + BM : p.S;  // chunk keys < chunk_hi are visible
  const int nch = (int)((chunk_hi + BN - 1) / BN);
  const int n = nct + nch;                                   // key tiles per sweep

  if (threadIdx.x == 0) {
    // consumer-side barriers of the softmax warpgroup take one arrival per thread
    for (int i = 0; i < kNumBars; ++i)
      mbar_init(bar(i), (i == B_S_EMPTY || i == B_S_EMPTY + 1 || i == B_P_FULL) ? 128u : 1u);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // =========================================================== TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_kc);
      prefetch_tmap(&tm_vc);
      mbar_arrive_expect_tx(bar(B_Q), kTile);
      const int zq = b * p.Hq + g;
      tma_load_3d(base + kOffQ, &tm_q, bar(B_Q), 0, (int)i0, zq);
      tma_load_3d(base + kOffQ + kAtom, &tm_q, bar(B_Q), 64, (int)i0, zq);
      int issued = 0;
      for (int it = 0; it < 2 * n; ++it) {
        const int stage = it % NS;
        const uint32_t ph = (uint32_t)(it / NS) & 1u;
        if (!mbar_wait(bar(B_KV_EMPTY + stage), ph ^ 1u, abort_flag, p.err, kWaitLimitNs, kErrTimeout))
          break;
        const bool sweep2 = it >= n;
        const int t = sweep2 ? it - n : it;
        const bool cache = t < nct;
        const CUtensorMap* mk = cache ? &tm_kc : &tm_k;
        const CUtensorMap* mv = cache ? &tm_vc : &tm_v;
        const int y = cache ? t * BN : (t - nct) * BN;
        const uint32_t dst = base + kOffKV + (uint32_t)stage * kStage;
        mbar_arrive_expect_tx(bar(B_KV_FULL + stage), sweep2 ? kStage : kTile);
        tma_load_3d(dst, mk, bar(B_KV_FULL + stage), 0, y, bh);
        tma_load_3d(dst + kAtom, mk, bar(B_KV_FULL + stage), 64, y, bh);
        if (sweep2) {
          tma_load_3d(dst + kTile, mv, bar(B_KV_FULL + stage), 0, y, bh);
          tma_load_3d(dst + kTile + kAtom, mv, bar(B_KV_FULL + stage), 64, y, bh);
        }
        issued = it + 1;
      }
      // drain: the last load of each stage has landed before the CTA may exit
      for (int it = issued - NS < 0 ? 0 : issued - NS; it < issued; ++it)
        mbar_wait(bar(B_KV_FULL + it % NS), (uint32_t)(it / NS) & 1u, abort_flag, p.err,
                  kWaitLimitNs, kErrTimeout);
    }
  } else if (warp == 1) {
    // =========================================================== MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16(128, 128, 0, 0);
      const uint32_t idesc_pv = idesc_bf16(128, 128, 1, 1);
      const uint32_t q_addr = base + kOffQ;
      const uint32_t p_addr = base + kOffP;
      bool ok = mbar_wait(bar(B_Q), 0, abort_flag, p.err, kWaitLimitNs, kErrTimeout);
      // issues S (sweep 1: Q K^T) or S^T (sweep 2: K Q^T) for iteration it
      auto issue_s = [&](int it) -> bool {
        const int stage = it % NS;
        const int sb = it & 1;
        if (!mbar_wait(bar(B_KV_FULL + stage), (uint32_t)(it / NS) & 1u, abort_flag, p.err,
                       kWaitLimitNs, kErrTimeout))
          return false;
        if (!mbar_wait(bar(B_S_EMPTY + sb), ((uint32_t)(it >> 1) & 1u) ^ 1u, abort_flag, p.err,
                       kWaitLimitNs, kErrTimeout))
          return false;
        tc_fence_after();
        const uint32_t k_addr = base + kOffKV + (uint32_t)stage * kStage;
        const uint32_t d_tmem = tmem + (uint32_t)sb * 128u;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * kAtom + (uint32_t)(kk & 3) * 32u;
          const uint64_t dq = smem_desc_sw128(q_addr + off, 16, 1024);
          const uint64_t dk = smem_desc_sw128(k_addr + off, 16, 1024);
          if (it < n) umma_bf16(d_tmem, dq, dk, idesc_s, kk > 0 ? 1u : 0u);
          else umma_bf16(d_tmem, dk, dq, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(B_S_FULL + sb));
        if (it < n) umma_commit(bar(B_KV_EMPTY + stage));   // sweep 1 only needs K
        return true;
      };
      for (int it = 0; ok && it < n; ++it) ok = issue_s(it);
      if (ok) ok = issue_s(n);
      for (int j = 0; ok && j < n; ++j) {
        const int it = n + j;
        if (j + 1 < n) ok = issue_s(it + 1);
        if (!ok) break;
        if (!mbar_wait(bar(B_P_FULL), (uint32_t)j & 1u, abort_flag, p.err, kWaitLimitNs, kErrTimeout)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int stage = it % NS;
        const uint32_t v_addr = base + kOffKV + (uint32_t)stage * kStage + kTile;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t dp = smem_desc_sw128(p_addr + (uint32_t)kk * 2048u, kAtom, 1024);
          const uint64_t dv = smem_desc_sw128(v_addr + (uint32_t)kk * 2048u, kAtom, 1024);
          umma_bf16(tmem + kColO, dp, dv, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar(B_P_EMPTY));
        umma_commit(bar(B_KV_EMPTY + stage));
      }
      umma_commit(bar(B_O_FULL));
      // every MMA issued has completed before TMEM is released
      umma_commit(bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0, abort_flag, p.err, kWaitLimitNs, kErrTimeout);
    }
  } else {
    // =========================================================== softmax / epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                 // TMEM lane owned by this thread
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const int64_t S = p.S, M = p.M, nv = p.n_valid;
    const float c = p.scale_log2;
    bool ok = true;

    // ----- sweep 1: thread = query row i0 + r
    const int64_t row_i = i0 + r;
    float m = -INFINITY, l = 0.f;
    for (int it = 0; ok && it < n; ++it) {
      const int sb = it & 1;
      // tcgen05.ld is warp-collective: the whole warp proceeds or stops together
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL + sb), (uint32_t)(it >> 1) & 1u,
                                             abort_flag, p.err, kWaitLimitNs, kErrTimeout));
      if (!ok) break;
      tc_fence_after();
      uint32_t v[4][32];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_ld32(lane_base + (uint32_t)sb * 128u + cc * 32, v[cc]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(B_S_EMPTY + sb));
      const bool cache = it < nct;
      const int64_t key0 = cache ? (int64_t)it * BN : (int64_t)(it - nct) * BN;
      // keys visible to this row: cache slots < n_valid; chunk keys <= row_i (and < S)
      const int64_t lim = cache ? nv : ((row_i + 1 < S) ? row_i + 1 : S);
      const int nvis = (int)(lim - key0 > BN ? BN : (lim - key0 < 0 ? 0 : lim - key0));
      float mx = -INFINITY;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float x = (cc * 32 + k < nvis) ? __uint_as_float(v[cc][k]) * c : -INFINITY;
          v[cc][k] = __float_as_uint(x);
          mx = fmaxf(mx, x);
        }
      if (mx > -INFINITY) {
        const float mn = fmaxf(m, mx);
        float sum = 0.f;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int k = 0; k < 32; ++k) sum += ex2(__uint_as_float(v[cc][k]) - mn);
        l = (m == -INFINITY ? 0.f : l * ex2(m - mn)) + sum;
        m = mn;
      }
      __syncwarp();
    }
    lse2[r] = (row_i < S && l > 0.f) ? m + lg2(l) : INFINITY;
    named_bar_sync(1, 128);

    // ----- sweep 2: thread = key (lane r of the S^T tile)
    float* part = p.partials + ((int64_t)bh * (p.G * p.n_rt) + (gl * p.n_rt + rt)) * (M + S);
    for (int j = 0; ok && j < n; ++j) {
      const int it = n + j;
      const int sb = it & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL + sb), (uint32_t)(it >> 1) & 1u,
                                             abort_flag, p.err, kWaitLimitNs, kErrTimeout));
      if (!ok) break;
      tc_fence_after();
      uint32_t v[4][32];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_ld32(lane_base + (uint32_t)sb * 128u + cc * 32, v[cc]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(B_S_EMPTY + sb));
      const bool cache = j < nct;
      const int64_t key = cache ? (int64_t)j * BN + r : (int64_t)(j - nct) * BN + r;
      const bool key_ok = cache ? key < nv : key < S;
      // chunk key `key` is seen by query columns q with i0 + q >= key
      const int qmin = cache ? 0 : (int)(key - i0 > 0 ? key - i0 : 0);
      float colsum = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        float ls[32];
#pragma unroll
        for (int k = 0; k < 32; k += 4) {
          const float4 t4 = *reinterpret_cast<const float4*>(lse2 + cc * 32 + k);
          ls[k] = t4.x; ls[k + 1] = t4.y; ls[k + 2] = t4.z; ls[k + 3] = t4.w;
        }
        float pv[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float x = fmaf(__uint_as_float(v[cc][k]), c, -ls[k]);
          const float e = ex2(x);
          pv[k] = (key_ok && cc * 32 + k >= qmin) ? e : 0.f;
          colsum += pv[k];
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) pk[cc * 16 + k] = pack_bf16(pv[2 * k], pv[2 * k + 1]);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_P_EMPTY), ((uint32_t)j & 1u) ^ 1u, abort_flag,
                                             p.err, kWaitLimitNs, kErrTimeout));
      if (!ok) break;
      // P^T row r (key) -> MN-major P tile: query block mb, 16-byte chunk cc8
      const uint32_t row_base = base + kOffP + (uint32_t)(r >> 3) * 1024u + (uint32_t)(r & 7) * 128u;
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const uint32_t mb = ch >> 3, c8 = ch & 7;
        const uint32_t addr = row_base + mb * kAtom + ((c8 ^ (uint32_t)(r & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[ch * 4]),
                     "r"(pk[ch * 4 + 1]), "r"(pk[ch * 4 + 2]), "r"(pk[ch * 4 + 3])
                     : "memory");
      }
      fence_async_smem();
      mbar_arrive(bar(B_P_FULL));
      if (key_ok) part[cache ? key : M + key] = colsum;
    }

    // ----- epilogue: thread = query row i0 + r
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_O_FULL), 0, abort_flag, p.err,
                                                   kWaitLimitNs, kErrTimeout));
    if (ok) {
      tc_fence_after();
      uint32_t o[4][32];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_ld32(lane_base + kColO + cc * 32, o[cc]);
      tmem_wait_ld();
      if (p.out != nullptr && row_i < S) {
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + (((int64_t)b * p.Hq + g) * S + row_i) * D;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int k = 0; k < 32; k += 8) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(o[cc][k]), __uint_as_float(o[cc][k + 1]));
            w.y = pack_bf16(__uint_as_float(o[cc][k + 2]), __uint_as_float(o[cc][k + 3]));
            w.z = pack_bf16(__uint_as_float(o[cc][k + 4]), __uint_as_float(o[cc][k + 5]));
            w.w = pack_bf16(__uint_as_float(o[cc][k + 6]), __uint_as_float(o[cc][k + 7]));
            *reinterpret_cast<uint4*>(orow + cc * 32 + k) = w;
          }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

cudaError_t get_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode ? cudaSuccess : cudaErrorNotSupported;
}

// [z][rows][D] bf16 tensor, box = 128 rows x 64 columns, 128-byte swizzle.
cudaError_t make_map(CUtensorMap* m, const void* ptr, int64_t rows, int64_t z) {
  if ((reinterpret_cast<uintptr_t>(ptr) & 15u) != 0) return cudaErrorMisalignedAddress;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)z};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)BM, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

bool attn_umma_supported(int dtype, int d) { return dtype == kBF16 && d == D; }

cudaError_t launch_attn_umma(const AttnArgs& a, cudaStream_t st) {
  if (a.d != D) return cudaErrorInvalidValue;
  cudaError_t e = get_encode();
  if (e != cudaSuccess) return e;
  CUtensorMap mq, mk, mv, mkc, mvc;
  const int64_t BHq = (int64_t)a.B * a.Hq, BHkv = (int64_t)a.B * a.Hkv;
  if ((e = make_map(&mq, a.q, a.S, BHq)) != cudaSuccess) return e;
  if ((e = make_map(&mk, a.k, a.S, BHkv)) != cudaSuccess) return e;
  if ((e = make_map(&mv, a.v, a.S, BHkv)) != cudaSuccess) return e;
  // with an empty cache the cache maps are never read; the chunk's stand in
  const bool has_cache = a.n_valid > 0;
  if ((e = make_map(&mkc, has_cache ? a.kc : a.k, has_cache ? a.M : a.S, BHkv)) != cudaSuccess) return e;
  if ((e = make_map(&mvc, has_cache ? a.vc : a.v, has_cache ? a.M : a.S, BHkv)) != cudaSuccess) return e;
  Params p;
  p.partials = a.partials;
  p.err = a.err;
  p.out = a.out;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.n_rt = (int)((a.S + BM - 1) / BM);
  p.S = a.S;
  p.M = a.M;
  p.n_valid = a.n_valid;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  e = cudaFuncSetAttribute(attn_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const int64_t grid = BHkv * p.G * p.n_rt;
  attn_umma_kernel<<<(unsigned)grid, kThreads, kSmemBytes, st>>>(mq, mk, mv, mkc, mvc, p);
  return cudaGetLastError();
}

}  // namespace h2o
