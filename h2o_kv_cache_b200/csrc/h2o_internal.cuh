// Internal interfaces between the C-ABI layer (h2o_api.cu) and the kernels.
// Nothing here is part of the public ABI (include/h2o.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

namespace h2o {

enum : int { kF32 = 0, kBF16 = 1 };

// Device error word bits (written by kernels, read back by the host).
enum : int {
  kErrTimeout = 1,      // a bounded mbarrier wait ran out
  kErrSelect = 2,       // fewer eligible slots than evictions needed
  kErrBounds = 4,       // an index check failed inside a kernel
};

// Summed attention weights are accumulated per (b, KV head) in one row of
// unsigned 64-bit fixed-point words, colacc[bh][c]: column c < M is cache slot
// c, c = M + j is chunk key j; rows are acc_stride words apart.  Every
// attention kernel adds its fp32 partial sums into the row with integer
// atomics: integer addition is exact and associative, so the result does not
// depend on the order in which CTAs finish (no float atomics, no partial rows
// for a separate reduction to read).  A value v is stored as
// round(v * 2^fx_shift) with fx_shift = 63 - bitlen(S * G): a column's total is
// at most S * G (each of the S * G query rows adds at most 1), so it fits in 63
// bits, and every fp32 partial at least 2^(24 - fx_shift) converts exactly.
// The reader converts the sum to fp32 once (correctly rounded) and clears the
// word, so the row is zero again before the next chunk's attention.
inline int colsum_shift(int64_t S, int G) {
  int64_t x = S * (int64_t)G;
  int bits = 0;
  while (x > 0) {
    ++bits;
    x >>= 1;
  }
  return 63 - bits;
}
#ifdef __CUDACC__
__device__ __forceinline__ void colsum_add(unsigned long long* p, float v, float fx_scale) {
  if (v > 0.f) atomicAdd(p, __float2ull_rn(v * fx_scale));
}
__device__ __forceinline__ unsigned long long colsum_fix(float v, float fx_scale) {
  return v > 0.f ? __float2ull_rn(v * fx_scale) : 0ull;
}
__device__ __forceinline__ float colsum_value(unsigned long long x, float fx_inv) {
  return __ull2float_rn(x) * fx_inv;
}
#endif
inline float fx_scale_of(int shift) { return std::ldexp(1.0f, shift); }
inline float fx_inv_of(int shift) { return std::ldexp(1.0f, -shift); }

struct AttnArgs {
  const void* q;      // [B, Hq, S, d]
  const void* k;      // [B, Hkv, S, d]
  const void* v;      // [B, Hkv, S, d]
  void* out;          // [B, Hq, S, d] or nullptr
  const void* kc;     // [B, Hkv, M, d]
  const void* vc;     // [B, Hkv, M, d]
  unsigned long long* colacc;   // [B * Hkv, acc_stride] fixed-point summed weights (zero on entry)
  int* err;           // device error word
  int B, Hq, Hkv, d;
  int64_t S, M, n_valid, acc_stride;
  float scale;        // 1/sqrt(d)
  int fx_shift;       // colsum_shift(S, Hq / Hkv)
  int split = 0;      // tensor-core kernel: CTAs per unit of work (0 = chosen by occupancy)
  int inject_timeout = 0;   // tensor-core kernel, test hook: one bounded wait runs out
};

// Row-tile height of each attention implementation.
constexpr int kSimtRowTile = 64;
constexpr int kUmmaRowTile = 128;

// Both kernels wait (griddepcontrol.wait) before their first global access, so
// with pdl they are launched as programmatic dependents of the stream's
// previous kernel and their prologue overlaps its last blocks.
cudaError_t launch_attn_simt(const AttnArgs& a, int dtype, bool pdl, cudaStream_t st);
cudaError_t launch_attn_umma(const AttnArgs& a, bool pdl, cudaStream_t st);
// The tensor-core kernel over n layers of identical sizes in one grid (layer
// after layer), 1 <= n <= attn_umma_max_group().
cudaError_t launch_attn_umma_group(const AttnArgs* a, int n, bool pdl, cudaStream_t st);
int attn_umma_max_group();
bool attn_umma_supported(int dtype, int d);

// Tensor-core attention as two persistent kernels over equal runs of all
// units' 256-key pairs (attn_stream.cu).  attn_stream_plan() sizes the run
// partition and the workspace for n_sm CTAs, or returns false when the
// partition does not fit (then the one-kernel path runs).
struct StreamPlan {
  int n_cta = 0, maxp = 0, units = 0;
  int heads_per_round = 1;   // (b, KV head) caches whose units a round partitions
  int64_t total_pairs = 0;
  size_t ml_bytes = 0, o_bytes = 0, count_bytes = 0;   // workspace the caller provides
};
bool attn_stream_plan(const AttnArgs& a, int n_sm, StreamPlan* plan);
cudaError_t launch_attn_stream(const AttnArgs& a, const StreamPlan& plan, void* ws_ml, void* ws_o,
                               int* count, bool pdl, cudaStream_t st);

// scores[b,h,c] += summed weight of column c (c < n_valid); newscore[b,h,j] =
// summed weight of chunk key j (j < S); the accumulator words read are cleared.
cudaError_t launch_score_reduce(unsigned long long* colacc, int64_t acc_stride, float fx_inv,
                                float* scores, float* newscore, int BH, int64_t S, int64_t M,
                                int64_t n_valid, cudaStream_t st);

// freed[bh, 0..S) = ascending evicted slots (need of them), then empty slots
// n_valid, n_valid + 1, ...  Sets kErrSelect in *err if a head has too few
// eligible slots.
// recency = 1 ranks the eligible slots by position alone (the lr policy).
cudaError_t launch_select(const float* scores, const int32_t* pos, int BH, int64_t M,
                          int64_t t0, int64_t R, int64_t need, int64_t n_valid, int64_t S,
                          int32_t* freed, int64_t freed_stride, int* err, cudaStream_t st,
                          int recency = 0);

// Chunk token i -> slot freed[bh, i]: K and V rows, pos = t0 + i, score = newscore[bh, i];
// evicted[bh, i] = the position the slot held before (-1 if it was empty).
cudaError_t launch_scatter(const void* k, const void* v, void* kc, void* vc, float* scores,
                           int32_t* pos, const int32_t* freed, const float* newscore,
                           int32_t* evicted, int BH, int64_t S, int64_t M, int d, int esize,
                           int64_t t0, cudaStream_t st);

// The three steps above as one launch: one thread-block cluster per (b, KV
// head).  freed[bh, 0..S) gets the same list launch_select writes.
struct TailArgs {
  unsigned long long* colacc;   // [BH, acc_stride] fixed-point summed weights (cleared here)
  float* scores;           // [BH, M]
  int32_t* pos;            // [BH, M]
  const uint4* k;          // chunk keys [BH, S, row_vecs]
  const uint4* v;          // chunk values [BH, S, row_vecs]
  uint4* kc;               // cache keys [BH, M, row_vecs]
  uint4* vc;               // cache values [BH, M, row_vecs]
  int32_t* freed;          // [BH, S]
  int32_t* evicted;        // [BH, S]: position each freed slot held before (-1: was empty)
  int* err;
  int64_t M, S, n_valid, t0, R, need, acc_stride;
  float fx_inv;            // 2^-fx_shift
  int recency;             // 1: rank eligible slots by position alone (lr policy)
  int row_vecs;
  int per, per_s;          // set by launch_tail
};
// Cluster size the fused tail runs with for these sizes (1 to 16), or 0
// if it cannot run (the caller then uses the three separate kernels); BH
// caches in all, in the one-layer kernel or (grouped) the kernel for groups.
int tail_cluster_size(int64_t M, int64_t S, int BH, bool grouped = false);
cudaError_t launch_tail(const TailArgs& a, int BH, int cs, bool pdl, cudaStream_t st);
// n layers of identical M and S in one launch (layer after layer),
// 1 <= n <= tail_max_group().
cudaError_t launch_tail_group(const TailArgs* a, int n, int BH, int cs, bool pdl, cudaStream_t st);
int tail_max_group();

// Chunks of a few tokens (G * S <= 16 query rows per KV head): attention with
// summed weights by FMA dot products over a key split (decode.cu).  Column
// sums go to the fixed-point accumulator row of each (b, KV head).
struct DecodeArgs {
  const void* q;        // [B, Hq, S, d]
  const void* k;        // [B, Hkv, S, d]
  const void* v;        // [B, Hkv, S, d]
  void* out;            // [B, Hq, S, d] or nullptr
  const void* kcache;   // [B, Hkv, M, d]
  const void* vcache;   // [B, Hkv, M, d]
  unsigned long long* colacc;   // [B * Hkv, acc_stride]
  int* err;
  int B, Hq, Hkv, G, d;
  int64_t S, M, n_valid, acc_stride;
  float scale_log2;     // log2(e) / sqrt(d)
  float fx_scale;       // 2^fx_shift
  int kc = 1;           // CTAs per cluster (set by launch_decode)
  int64_t per = 0;      // keys per CTA (set by launch_decode)
};
bool decode_supported(int G, int64_t S, int64_t keys);
cudaError_t launch_decode(DecodeArgs a, int dtype, int BH, bool pdl, cudaStream_t st);

// Records msg as this thread's last error (h2o_last_error(NULL)); returns code.
int set_thread_error(int code, const char* msg);

}  // namespace h2o
