// Device and host pieces shared by the tensor-core attention kernels
// (attn_umma.cu: both sweeps in one kernel; attn_stream.cu: one kernel per
// sweep over balanced runs of key tiles).  Included by those files only.
//
// "Learning how to Forget: Fine-tuning for Long-Context Sparse Attention",
// FAQ answer 3 (SDPA that also returns the summed attention weights).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "h2o_internal.cuh"
#include "sm100.cuh"

namespace h2o {
namespace attn {

using namespace sm100;

constexpr int BM = kUmmaRowTile;   // query rows per head per CTA
constexpr int BN = 128;            // keys per TMA tile
constexpr int D = 128;             // head dimension
constexpr uint32_t kAtom = 128 * 64 * 2;         // [128 rows x 64 bf16] box: 16 KB
constexpr uint32_t kTile = 2 * kAtom;            // [128 x 128] bf16: 32 KB

// Sweep-2 ring positions: the K / V tiles enter in the order the MMAs use
// them -- K0, K1, V0, K2, V1, ..., K(n-1), V(n-2), V(n-1).
__device__ __forceinline__ int k_pos(int j) { return j == 0 ? 0 : 2 * j - 1; }
__device__ __forceinline__ int v_pos(int n, int j) { return j + 1 < n ? 2 * j + 2 : 2 * j + 1; }

// Offset of k-step kk (16 columns) inside a K-major tile of `rows` rows whose
// two 64-column atoms are rows * 128 bytes apart.
__device__ __forceinline__ uint32_t kmajor_off(int kk, uint32_t rows) {
  return (uint32_t)(kk >> 2) * rows * 128u + (uint32_t)(kk & 3) * 32u;
}

// Sweep 1: one 64-key chunk of a row (x = raw scores in v, nvis of them
// visible) folded into the running (m, l), base 2.
__device__ __forceinline__ void row_chunk(uint32_t (&v)[2][32], int nvis, float c, float& m, float& l) {
  if (nvis < 64) {
#pragma unroll
    for (int k = 0; k < 64; ++k)
      if (k >= nvis) v[k >> 5][k & 31] = __float_as_uint(-INFINITY);
  }
  float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  float s8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const float nm = -m;
#pragma unroll
  for (int k = 0; k < 64; ++k) {
    const float x = __uint_as_float(v[k >> 5][k & 31]);
    mx4[k & 3] = fmaxf(mx4[k & 3], x);
    s8[k & 7] += ex2(fmaf(x, c, nm));
  }
  const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * c;
  if (mx > m + 8.f) {
    // rare: raise the reference and recompute this chunk's sum against it
#pragma unroll
    for (int k = 0; k < 8; ++k) s8[k] = 0.f;
#pragma unroll
    for (int k = 0; k < 64; ++k) s8[k & 7] += ex2(fmaf(__uint_as_float(v[k >> 5][k & 31]), c, -mx));
    l = (m == -INFINITY) ? 0.f : l * ex2(m - mx);
    m = mx;
  }
  l += ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
}

// Sweep 2: 64 query columns of a key's S^T row -> p = 2^(s c - lse) (zero where
// masked), column-sum terms into cs8, packed bf16 pairs into pk.
template <bool kFull>
__device__ __forceinline__ void key_half(const uint32_t (&v)[2][32], const float* nl, float c,
                                         bool key_ok, int qmin, float (&cs8)[8], uint32_t (&pk)[32]) {
#pragma unroll
  for (int k = 0; k < 64; k += 4) {
    const float4 n4 = *reinterpret_cast<const float4*>(nl + k);
    const float nlk[4] = {n4.x, n4.y, n4.z, n4.w};
    float e[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      e[i] = ex2(fmaf(__uint_as_float(v[(k + i) >> 5][(k + i) & 31]), c, nlk[i]));
      if (!kFull) e[i] = (key_ok && k + i >= qmin) ? e[i] : 0.f;
      cs8[(k + i) & 7] += e[i];
    }
    pk[k >> 1] = pack_bf16(e[0], e[1]);
    pk[(k >> 1) + 1] = pack_bf16(e[2], e[3]);
  }
}

// Sweep 2: a key's 64-query half of P^T (packed) into its 128-byte swizzled row.
__device__ __forceinline__ void store_p_half(uint32_t row_addr, int r, const uint32_t (&pk)[32]) {
#pragma unroll
  for (int c8 = 0; c8 < 8; ++c8) {
    const uint32_t addr = row_addr + ((((uint32_t)c8) ^ (uint32_t)(r & 7)) << 4);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[c8 * 4]),
                 "r"(pk[c8 * 4 + 1]), "r"(pk[c8 * 4 + 2]), "r"(pk[c8 * 4 + 3])
                 : "memory");
  }
}

// ---------------------------------------------------------------- host side
inline PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
inline std::once_flag g_encode_once;

inline cudaError_t get_encode() {
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
inline cudaError_t make_map(CUtensorMap* m, const void* ptr, int64_t rows, int64_t z) {
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


}  // namespace attn
}  // namespace h2o
