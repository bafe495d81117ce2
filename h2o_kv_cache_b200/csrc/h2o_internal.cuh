// Internal interfaces between the C-ABI layer (h2o_api.cu) and the kernels.
// Nothing here is part of the public ABI (include/h2o.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace h2o {

enum : int { kF32 = 0, kBF16 = 1 };

// Device error word bits (written by kernels, read back by the host).
enum : int {
  kErrTimeout = 1,      // a bounded mbarrier wait ran out
  kErrSelect = 2,       // fewer eligible slots than evictions needed
  kErrBounds = 4,       // an index check failed inside a kernel
};

// One chunk's attention with summed weights, for all (b, KV head) of a layer.
// Column c of a partial row: c < M is cache slot c, c = M + j is chunk key j.
// Partial row tq of a (b, h) group belongs to query-row tile (local head gl,
// row tile rt): tq = gl * n_rt + rt, n_rt = ceil(S / row_tile).  A tile writes
// every cache column < n_valid and the chunk columns of keys it can see
// (key j < min(S, (rt + 1) * row_tile)).
struct AttnArgs {
  const void* q;      // [B, Hq, S, d]
  const void* k;      // [B, Hkv, S, d]
  const void* v;      // [B, Hkv, S, d]
  void* out;          // [B, Hq, S, d] or nullptr
  const void* kc;     // [B, Hkv, M, d]
  const void* vc;     // [B, Hkv, M, d]
  float* partials;    // [B, Hkv, G * n_rt, M + S]
  int* err;           // device error word
  int B, Hq, Hkv, d;
  int64_t S, M, n_valid;
  float scale;        // 1/sqrt(d)
};

// Row-tile height of each attention implementation (sets the partials layout).
constexpr int kSimtRowTile = 64;
constexpr int kUmmaRowTile = 128;

cudaError_t launch_attn_simt(const AttnArgs& a, int dtype, cudaStream_t st);
cudaError_t launch_attn_umma(const AttnArgs& a, cudaStream_t st);
bool attn_umma_supported(int dtype, int d);

// scores[b,h,c] += sum of partial column c (c < n_valid);
// newscore[b,h,j] = sum of partial column M + j (j < S).
cudaError_t launch_score_reduce(const float* partials, float* scores, float* newscore, int BH,
                                int G, int64_t S, int64_t M, int64_t n_valid, int row_tile,
                                cudaStream_t st);

// freed[bh, 0..S) = ascending evicted slots (need of them), then empty slots
// n_valid, n_valid + 1, ...  Sets kErrSelect in *err if a head has too few
// eligible slots.
cudaError_t launch_select(const float* scores, const int32_t* pos, int BH, int64_t M,
                          int64_t t0, int64_t R, int64_t need, int64_t n_valid, int64_t S,
                          int32_t* freed, int64_t freed_stride, int* err, cudaStream_t st);

// Chunk token i -> slot freed[bh, i]: K and V rows, pos = t0 + i, score = newscore[bh, i].
cudaError_t launch_scatter(const void* k, const void* v, void* kc, void* vc, float* scores,
                           int32_t* pos, const int32_t* freed, const float* newscore, int BH,
                           int64_t S, int64_t M, int d, int esize, int64_t t0, cudaStream_t st);

// Records msg as this thread's last error (h2o_last_error(NULL)); returns code.
int set_thread_error(int code, const char* msg);

}  // namespace h2o
