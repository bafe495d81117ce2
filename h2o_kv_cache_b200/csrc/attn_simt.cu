// SIMT attention with summed attention weights (fp32 arithmetic).
//
// The float32 path of the library (a TF32 tensor-core product would exceed the
// 1e-4 relative output bound of float32 parity), and the bf16 path for head
// sizes the tensor-core kernel does not cover.
//
// "Learning how to Forget: Fine-tuning for Long-Context Sparse Attention",
// FAQ answer 3: SDPA that also returns the summed attention weights; §1 ¶1:
// attention over a fixed-size cache.  Each query row sees the valid cache
// slots [0, n_valid) plus the chunk keys j <= i.
//
// One block = 64 query rows of one query head, one thread per row.  Two sweeps
// over the visible keys: the first finds each row's log-sum-exp, the second
// forms the exact probabilities p = exp(s - lse), accumulates out = p.V and
// adds the block's column sums of p to the (b, KV head)'s accumulator row.
#include "h2o_internal.cuh"

namespace h2o {
namespace {

constexpr int BR = kSimtRowTile;  // query rows per block
constexpr int BK = 64;            // keys per tile

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f(float x, float* p) { *p = x; }
__device__ __forceinline__ void from_f(float x, __nv_bfloat16* p) { *p = __float2bfloat16_rn(x); }

template <typename T, int D>
__global__ void __launch_bounds__(BR) attn_simt_kernel(AttnArgs a) {
  extern __shared__ float smem[];
  float* Qs = smem;                  // [BR][D + 1]
  float* Ks = Qs + BR * (D + 1);     // [BK][D]
  float* Vs = Ks + BK * D;           // [BK][D]
  float* Ps = Vs + BK * D;           // [BR][BK + 1]

  const int tid = threadIdx.x;
  const int rt = blockIdx.x;
  const int g = blockIdx.y;
  const int b = blockIdx.z;
  const int G = a.Hq / a.Hkv;
  const int h = g / G;
  const int64_t S = a.S, M = a.M, nv = a.n_valid;
  const int64_t i0 = (int64_t)rt * BR;
  const int64_t i = i0 + tid;
  const bool row_ok = i < S;

  const T* qb = static_cast<const T*>(a.q) + ((int64_t)b * a.Hq + g) * S * D;
  const T* kb = static_cast<const T*>(a.k) + ((int64_t)b * a.Hkv + h) * S * D;
  const T* vb = static_cast<const T*>(a.v) + ((int64_t)b * a.Hkv + h) * S * D;
  const T* kcb = static_cast<const T*>(a.kc) + ((int64_t)b * a.Hkv + h) * M * D;
  const T* vcb = static_cast<const T*>(a.vc) + ((int64_t)b * a.Hkv + h) * M * D;
  unsigned long long* acc_row = a.colacc + ((int64_t)b * a.Hkv + h) * a.acc_stride;
  const float fx_scale = __int_as_float((127 + a.fx_shift) << 23);   // 2^fx_shift

  // the cache and the accumulator row may still be in use by the previous kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");

  for (int e = tid; e < BR * D; e += BR) {
    const int r = e / D, c = e - r * D;
    const int64_t ii = i0 + r;
    Qs[r * (D + 1) + c] = ii < S ? to_f(qb[ii * D + c]) : 0.f;
  }

  // key tiles: cache tiles first, then the chunk tiles this block can see
  const int64_t n_ct_cache = (nv + BK - 1) / BK;
  const int64_t chunk_hi = (i0 + BR < S) ? (i0 + BR) : S;   // chunk keys < chunk_hi
  const int64_t n_ct_chunk = (chunk_hi + BK - 1) / BK;
  const int64_t n_tiles = n_ct_cache + n_ct_chunk;
  const float scale = a.scale;

  float m = -INFINITY, l = 0.f;
  for (int pass = 0; pass < 2; ++pass) {
    const float lse = (row_ok && l > 0.f) ? m + logf(l) : INFINITY;
    float acc[D];
#pragma unroll
    for (int c = 0; c < D; ++c) acc[c] = 0.f;

    for (int64_t t = 0; t < n_tiles; ++t) {
      const bool is_cache = t < n_ct_cache;
      const int64_t key0 = is_cache ? t * BK : (t - n_ct_cache) * BK;
      const int64_t key_lim = is_cache ? nv : chunk_hi;
      const T* ksrc = is_cache ? kcb : kb;
      const T* vsrc = is_cache ? vcb : vb;
      __syncthreads();
      for (int e = tid; e < BK * D; e += BR) {
        const int r = e / D, c = e - r * D;
        const int64_t kk = key0 + r;
        const bool ok = kk < key_lim;
        Ks[e] = ok ? to_f(ksrc[kk * D + c]) : 0.f;
        if (pass == 1) Vs[e] = ok ? to_f(vsrc[kk * D + c]) : 0.f;
      }
      __syncthreads();

      float s[BK];
      float tmax = -INFINITY;
#pragma unroll 4
      for (int j = 0; j < BK; ++j) {
        const int64_t kk = key0 + j;
        const bool vis = row_ok && kk < key_lim && (is_cache || kk <= i);
        float dot = 0.f;
#pragma unroll 16
        for (int c = 0; c < D; ++c) dot = fmaf(Qs[tid * (D + 1) + c], Ks[j * D + c], dot);
        s[j] = vis ? dot * scale : -INFINITY;
        tmax = fmaxf(tmax, s[j]);
      }
      if (pass == 0) {
        if (tmax > -INFINITY) {
          const float mn = fmaxf(m, tmax);
          float sum = 0.f;
#pragma unroll 8
          for (int j = 0; j < BK; ++j) sum += expf(s[j] - mn);
          l = l * expf(m - mn) + sum;
          m = mn;
        }
      } else {
#pragma unroll 4
        for (int j = 0; j < BK; ++j) {
          const float p = expf(s[j] - lse);   // 0 for masked keys and rows
          Ps[tid * (BK + 1) + j] = p;
#pragma unroll 16
          for (int c = 0; c < D; ++c) acc[c] = fmaf(p, Vs[j * D + c], acc[c]);
        }
        __syncthreads();
        // column sums of this tile over the block's rows (thread = key)
        const int64_t kk = key0 + tid;
        if (kk < key_lim) {
          float cs = 0.f;
          for (int r = 0; r < BR; ++r) cs += Ps[r * (BK + 1) + tid];
          colsum_add(acc_row + (is_cache ? kk : M + kk), cs, fx_scale);
        }
      }
    }
    if (pass == 1 && row_ok && a.out != nullptr) {
      T* ob = static_cast<T*>(a.out) + (((int64_t)b * a.Hq + g) * S + i) * D;
#pragma unroll
      for (int c = 0; c < D; ++c) from_f(acc[c], ob + c);
    }
  }
}

template <typename T, int D>
cudaError_t launch_t(const AttnArgs& a, bool pdl, cudaStream_t st) {
  const size_t smem = sizeof(float) * (BR * (D + 1) + 2 * BK * D + BR * (BK + 1));
  auto kern = attn_simt_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((a.S + BR - 1) / BR), (unsigned)a.Hq, (unsigned)a.B);
  cfg.blockDim = dim3(BR);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace

cudaError_t launch_attn_simt(const AttnArgs& a, int dtype, bool pdl, cudaStream_t st) {
  if (dtype == kF32) {
    if (a.d == 64) return launch_t<float, 64>(a, pdl, st);
    if (a.d == 128) return launch_t<float, 128>(a, pdl, st);
  } else {
    if (a.d == 64) return launch_t<__nv_bfloat16, 64>(a, pdl, st);
    if (a.d == 128) return launch_t<__nv_bfloat16, 128>(a, pdl, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace h2o
