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
// Column c of a partial row: c < M is cache slot c, c = M + j is chunk key j;
// rows are part_stride floats apart (M + S rounded up to a multiple of 4, so
// every row starts 16-byte aligned).  Partial row tq of a (b, h) group belongs
// to (group gl, row tile rt): tq = gl * n_rt + rt, n_rt = ceil(S / row_tile).
// A group is one query head of the KV head's G in the SIMT kernel, and a pair
// of them (heads 2gl and 2gl + 1, summed) in the tensor-core kernel; see
// partial_groups().  A tile writes every cache column < n_valid and the chunk
// columns of keys it can see (key j < min(S, (rt + 1) * row_tile)).
inline int64_t partial_stride(int64_t M, int64_t S) { return (M + S + 3) & ~(int64_t)3; }
inline int partial_groups(int G, bool umma) { return umma ? (G + 1) / 2 : G; }
// The stream-partitioned tensor-core path writes one partial row per softmax
// warpgroup: kStreamRows per head pair (its four 64-query slices).
constexpr int kStreamRows = 4;
inline int stream_partial_groups(int G) { return kStreamRows * ((G + 1) / 2); }

// Order in which a column's partial rows are added, shared by both tail paths
// so they agree bit for bit: the column's list of n rows (for a chunk column,
// the rows that wrote it, group-major) is cut into kQuarters contiguous runs,
// run q = [q * n / kQuarters, (q + 1) * n / kQuarters); each run is summed in
// order starting from 0, and then the run sums are added in order.
constexpr int kQuarters = 4;

struct AttnArgs {
  const void* q;      // [B, Hq, S, d]
  const void* k;      // [B, Hkv, S, d]
  const void* v;      // [B, Hkv, S, d]
  void* out;          // [B, Hq, S, d] or nullptr
  const void* kc;     // [B, Hkv, M, d]
  const void* vc;     // [B, Hkv, M, d]
  float* partials;    // [B, Hkv, partial_groups * n_rt, part_stride]
  int* err;           // device error word
  int B, Hq, Hkv, d;
  int64_t S, M, n_valid, part_stride;
  float scale;        // 1/sqrt(d)
  int split = 0;      // tensor-core kernel: CTAs per unit of work (0 = chosen by occupancy)
  int inject_timeout = 0;   // tensor-core kernel, test hook: one bounded wait runs out
};

// Row-tile height of each attention implementation (sets the partials layout).
constexpr int kSimtRowTile = 64;
constexpr int kUmmaRowTile = 128;

// Both kernels wait (griddepcontrol.wait) before their first global access, so
// with pdl they are launched as programmatic dependents of the stream's
// previous kernel and their prologue overlaps its last blocks.
cudaError_t launch_attn_simt(const AttnArgs& a, int dtype, bool pdl, cudaStream_t st);
cudaError_t launch_attn_umma(const AttnArgs& a, bool pdl, cudaStream_t st);
bool attn_umma_supported(int dtype, int d);

// Tensor-core attention as two persistent kernels over equal runs of all
// units' 256-key pairs (attn_stream.cu).  attn_stream_plan() sizes the run
// partition and the workspace for n_sm CTAs, or returns false when the
// partition does not fit (then the one-kernel path runs).
struct StreamPlan {
  int n_cta = 0, maxp = 0, units = 0;
  int64_t total_pairs = 0;
  size_t ml_bytes = 0, o_bytes = 0, count_bytes = 0;   // workspace the caller provides
};
bool attn_stream_plan(const AttnArgs& a, int n_sm, StreamPlan* plan);
cudaError_t launch_attn_stream(const AttnArgs& a, const StreamPlan& plan, void* ws_ml, void* ws_o,
                               int* count, bool pdl, cudaStream_t st);

// scores[b,h,c] += sum of partial column c (c < n_valid);
// newscore[b,h,j] = sum of partial column M + j (j < S); n_grp partial groups.
cudaError_t launch_score_reduce(const float* partials, float* scores, float* newscore, int BH,
                                int n_grp, int64_t S, int64_t M, int64_t n_valid, int row_tile,
                                int64_t part_stride, cudaStream_t st);

// freed[bh, 0..S) = ascending evicted slots (need of them), then empty slots
// n_valid, n_valid + 1, ...  Sets kErrSelect in *err if a head has too few
// eligible slots.
cudaError_t launch_select(const float* scores, const int32_t* pos, int BH, int64_t M,
                          int64_t t0, int64_t R, int64_t need, int64_t n_valid, int64_t S,
                          int32_t* freed, int64_t freed_stride, int* err, cudaStream_t st);

// Chunk token i -> slot freed[bh, i]: K and V rows, pos = t0 + i, score = newscore[bh, i];
// evicted[bh, i] = the position the slot held before (-1 if it was empty).
cudaError_t launch_scatter(const void* k, const void* v, void* kc, void* vc, float* scores,
                           int32_t* pos, const int32_t* freed, const float* newscore,
                           int32_t* evicted, int BH, int64_t S, int64_t M, int d, int esize,
                           int64_t t0, cudaStream_t st);

// The three steps above as one launch: one thread-block cluster per (b, KV
// head).  freed[bh, 0..S) gets the same list launch_select writes.
struct TailArgs {
  const float* partials;   // [BH, n_grp * n_rt, stride]
  float* scores;           // [BH, M]
  int32_t* pos;            // [BH, M]
  const uint4* k;          // chunk keys [BH, S, row_vecs]
  const uint4* v;          // chunk values [BH, S, row_vecs]
  uint4* kc;               // cache keys [BH, M, row_vecs]
  uint4* vc;               // cache values [BH, M, row_vecs]
  int32_t* freed;          // [BH, S]
  int32_t* evicted;        // [BH, S]: position each freed slot held before (-1: was empty)
  int* err;
  int64_t M, S, n_valid, t0, R, need, stride;
  int n_grp, n_rt, row_tile, row_vecs;
  int per, per_s;          // set by launch_tail
};
// Cluster size the fused tail runs with for these sizes (16, 8, ..., 1), or 0
// if it cannot run (the caller then uses the three separate kernels).
int tail_cluster_size(int64_t M, int64_t S, int BH);
cudaError_t launch_tail(const TailArgs& a, int BH, int cs, bool pdl, cudaStream_t st);

// Chunks of a few tokens (G * S <= 16 query rows per KV head): attention with
// summed weights by FMA dot products over a key split (decode.cu).  Column
// sums go to ONE partial row per (b, KV head): partials [BH][stride].
struct DecodeArgs {
  const void* q;        // [B, Hq, S, d]
  const void* k;        // [B, Hkv, S, d]
  const void* v;        // [B, Hkv, S, d]
  void* out;            // [B, Hq, S, d] or nullptr
  const void* kcache;   // [B, Hkv, M, d]
  const void* vcache;   // [B, Hkv, M, d]
  float* partials;      // [B * Hkv, stride]
  int* err;
  int B, Hq, Hkv, G, d;
  int64_t S, M, n_valid, stride;
  float scale_log2;     // log2(e) / sqrt(d)
  int kc = 1;           // CTAs per cluster (set by launch_decode)
  int64_t per = 0;      // keys per CTA (set by launch_decode)
};
bool decode_supported(int G, int64_t S, int64_t keys);
cudaError_t launch_decode(DecodeArgs a, int dtype, int BH, bool pdl, cudaStream_t st);

// Records msg as this thread's last error (h2o_last_error(NULL)); returns code.
int set_thread_error(int code, const char* msg);

}  // namespace h2o
