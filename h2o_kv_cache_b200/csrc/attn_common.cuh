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

// 2^x on the FMA pipe for a packed pair, each x <= 2^22; x below -126 (and
// NaN) is taken as -126, which gives a value of at most 2^-126 (a denormal or
// the smallest normal: with the cubic's value just under 1 a lower exponent
// would wrap into the sign bit).  Cody-Waite range reduction:
// 2^x = 2^j * 2^f with j = floor(x) and f = x - j in [0, 1), both exact; 2^f
// by a cubic whose coefficients minimise the largest relative error over
// [0, 1) (a weighted least-squares fit iterated towards equal ripple; max
// relative error 7.5e-5, mean 5e-6); the exponent j is added to the bits of
// the cubic's value.  Adding 1.5 * 2^23 rounded towards -inf leaves floor(x)
// in the low mantissa bits of t, so (bits(t) << 23) is j << 23 modulo 2^32.
__device__ __forceinline__ void ex2_poly2(uint64_t x2, float& r0, float& r1) {
  float a, b;
  f2_unpack(x2, a, b);
  const uint64_t x = f2_pack(fmaxf(a, -126.f), fmaxf(b, -126.f));
  const uint64_t magic = f2_pack(12582912.f, 12582912.f);
  const uint64_t t = fadd2_rm(x, magic);
  const uint64_t f = fsub2(x, fsub2(t, magic));
  uint64_t q = ffma2(f2_pack(0.078023761510849f, 0.078023761510849f), f,
                     f2_pack(0.22606682777404785f, 0.22606682777404785f));
  q = ffma2(q, f, f2_pack(0.6958343982696533f, 0.6958343982696533f));
  q = ffma2(q, f, f2_pack(0.9999250173568726f, 0.9999250173568726f));
  float q0, q1, t0, t1;
  f2_unpack(q, q0, q1);
  f2_unpack(t, t0, t1);
  r0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
  r1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
}

// Which exponentials run on the FMA pipe: the pair (k, k + 1), k even, of a
// row or column uses ex2_poly2 when bit (k / 2) % 4 of the mask is set, the
// MUFU unit otherwise.  The MUFU unit does 16 exponentials per clock per SM;
// moving a quarter of them to the FMA pipe unloads it at the cost of about
// five extra instructions each.
#ifndef H2O_EMU1
#define H2O_EMU1 0x8
#endif
#ifndef H2O_EMU2
#define H2O_EMU2 0x8
#endif
constexpr unsigned kEmuRow = H2O_EMU1;   // sweep 1 (row sums)
constexpr unsigned kEmuKey = H2O_EMU2;   // sweep 2 (probabilities and column sums)

template <unsigned kMask>
__device__ __forceinline__ void ex2_pair(uint64_t x2, int k, float& r0, float& r1) {
  if ((kMask >> ((k >> 1) & 3)) & 1u) {
    ex2_poly2(x2, r0, r1);
  } else {
    float a, b;
    f2_unpack(x2, a, b);
    r0 = ex2(a);
    r1 = ex2(b);
  }
}

// Sweep 1: one 64-key chunk of a row (x = raw scores in v, nvis of them
// visible) folded into the running (m, l), base 2.  Pairs of elements go
// through the two-lane instructions; the eight partial sums are the lanes of
// four packed accumulators.
__device__ __forceinline__ void row_chunk(uint32_t (&v)[2][32], int nvis, float c, float& m, float& l) {
  if (nvis < 64) {
#pragma unroll
    for (int k = 0; k < 64; ++k)
      if (k >= nvis) v[k >> 5][k & 31] = __float_as_uint(-INFINITY);
  }
  float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  uint64_t s4[4] = {0ull, 0ull, 0ull, 0ull};
  const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(-m, -m);
#pragma unroll
  for (int k = 0; k < 64; k += 2) {
    const float x0 = __uint_as_float(v[k >> 5][k & 31]), x1 = __uint_as_float(v[k >> 5][(k & 31) + 1]);
    mx4[(k >> 1) & 3] = fmax3(mx4[(k >> 1) & 3], x0, x1);
    float e0, e1;
    ex2_pair<kEmuRow>(ffma2(f2_pack(x0, x1), c2, nm2), k, e0, e1);
    s4[(k >> 1) & 3] = fadd2(s4[(k >> 1) & 3], f2_pack(e0, e1));
  }
  const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * c;
  float s8[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) f2_unpack(s4[i], s8[2 * i], s8[2 * i + 1]);
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

// Sweep 2: kN query columns of a key's S^T row (x = raw scores in v) ->
// p = 2^(s c - lse) (zero where masked), column-sum terms into the packed
// accumulators cs4 (lane i of cs4[j] holds the terms of columns = 2j + i
// mod 8), packed bf16 pairs into pk[0 .. kN/2).
template <bool kFull, int kN>
__device__ __forceinline__ void key_part(const uint32_t* v, const float* nl, float c, bool key_ok,
                                         int qmin, uint64_t (&cs4)[4], uint32_t* pk) {
  const uint64_t c2 = f2_pack(c, c);
#pragma unroll
  for (int k = 0; k < kN; k += 4) {
    const float4 n4 = *reinterpret_cast<const float4*>(nl + k);
    float e[4];
    ex2_pair<kEmuKey>(ffma2(f2_pack(__uint_as_float(v[k]), __uint_as_float(v[k + 1])), c2,
                            f2_pack(n4.x, n4.y)), k, e[0], e[1]);
    ex2_pair<kEmuKey>(ffma2(f2_pack(__uint_as_float(v[k + 2]), __uint_as_float(v[k + 3])), c2,
                            f2_pack(n4.z, n4.w)), k + 2, e[2], e[3]);
    if (!kFull) {
#pragma unroll
      for (int i = 0; i < 4; ++i) e[i] = (key_ok && k + i >= qmin) ? e[i] : 0.f;
    }
    cs4[(k >> 1) & 3] = fadd2(cs4[(k >> 1) & 3], f2_pack(e[0], e[1]));
    cs4[((k >> 1) + 1) & 3] = fadd2(cs4[((k >> 1) + 1) & 3], f2_pack(e[2], e[3]));
    pk[k >> 1] = pack_bf16(e[0], e[1]);
    pk[(k >> 1) + 1] = pack_bf16(e[2], e[3]);
  }
}

// The same for a 64-query half held as two 32-column TMEM loads.
template <bool kFull>
__device__ __forceinline__ void key_half(const uint32_t (&v)[2][32], const float* nl, float c,
                                         bool key_ok, int qmin, uint64_t (&cs4)[4], uint32_t (&pk)[32]) {
  key_part<kFull, 32>(v[0], nl, c, key_ok, qmin, cs4, pk);
  key_part<kFull, 32>(v[1], nl + 32, c, key_ok, qmin - 32, cs4, pk + 16);
}

// The column sum of a key: the eight partial sums in a fixed order.
__device__ __forceinline__ float cs_total(const uint64_t (&cs4)[4]) {
  float s[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) f2_unpack(cs4[i], s[2 * i], s[2 * i + 1]);
  return ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
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
