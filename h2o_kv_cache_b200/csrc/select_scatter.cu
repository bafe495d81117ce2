// Score accumulation, masked selection of the slots to evict, and the scatter
// of the chunk's K/V into the freed slots.
//
// "Learning how to Forget: Fine-tuning for Long-Context Sparse Attention",
// §1 Introduction ¶1 (fixed-size cache, slots evicted once full) and ¶4 (H2O,
// the heavy-hitter oracle: the running sum of summed attention weights ranks
// the slots); Figure 1(c) (per-chunk buffer deltas: the evicted slots and the
// new K/V rows written into them).
#include "h2o_internal.cuh"

namespace h2o {
namespace {

// ---------------------------------------------------------------------------
// Score accumulation: each column's summed weight from the fixed-point
// accumulator row (the word is cleared for the next chunk).
// ---------------------------------------------------------------------------
__global__ void score_reduce_kernel(unsigned long long* __restrict__ colacc, int64_t acc_stride,
                                    float fx_inv, float* __restrict__ scores,
                                    float* __restrict__ newscore, int64_t S, int64_t M,
                                    int64_t n_valid) {
  const int bh = blockIdx.y;
  const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= n_valid + S) return;
  unsigned long long* acc = colacc + (int64_t)bh * acc_stride;
  const int64_t col = c < n_valid ? c : M + (c - n_valid);
  const float v = colsum_value(acc[col], fx_inv);
  acc[col] = 0ull;
  if (c < n_valid) scores[(int64_t)bh * M + c] += v;
  else newscore[(int64_t)bh * S + (c - n_valid)] = v;
}

// ---------------------------------------------------------------------------
// Selection.  Each slot gets a 64-bit key: order-preserving bits of its score
// in the high word, its token position in the low word, so ascending keys are
// ascending (score, pos) -- the older token goes first on equal scores.  An
// MSD radix select (8 bits a pass) finds the need-th smallest key among the
// eligible slots (valid and pos < t0 - R); every eligible slot whose key is at
// or below it is evicted, written out in ascending slot order.
// ---------------------------------------------------------------------------
constexpr int kSelThreads = 1024;

__device__ __forceinline__ uint32_t ordered_bits(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kSelThreads)
select_kernel(const float* __restrict__ scores, const int32_t* __restrict__ pos, int64_t M,
              int64_t t0, int64_t R, int64_t need, int64_t n_valid, int64_t S,
              int32_t* __restrict__ freed, int64_t freed_stride, int* err, int recency) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_tot[kSelThreads / 32];
  __shared__ uint64_t sh_prefix, sh_mask;
  __shared__ int64_t sh_kth;
  __shared__ int sh_done;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x;
  const float* sc = scores + (int64_t)bh * M;
  const int32_t* ps = pos + (int64_t)bh * M;
  int32_t* out = freed + (int64_t)bh * freed_stride;
  const int64_t lim = t0 - R;   // eligible: 0 <= pos < lim

  if (tid == 0) { sh_prefix = 0; sh_mask = 0; sh_kth = need; sh_done = (need == 0); }
  __syncthreads();

  for (int shift = 56; shift >= 0 && !sh_done; shift -= 8) {
    for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    const uint64_t prefix = sh_prefix, mask = sh_mask;
    for (int64_t base = 0; base < M; base += kSelThreads) {
      const int64_t s = base + tid;
      bool take = false;
      uint32_t digit = 0;
      if (s < M) {
        const int32_t p = ps[s];
        if (p >= 0 && p < lim) {
          const uint64_t key = (recency ? 0ull : (uint64_t)ordered_bits(sc[s]) << 32) | (uint32_t)p;
          if ((key & mask) == prefix) { take = true; digit = (uint32_t)(key >> shift) & 0xFFu; }
        }
      }
      // warp-aggregated histogram update
      const unsigned active = __ballot_sync(0xffffffffu, take);
      if (take) {
        const unsigned peers = __match_any_sync(active, digit);
        if ((__ffs(peers) - 1) == lane) atomicAdd(&hist[digit], (uint32_t)__popc(peers));
      }
    }
    __syncthreads();
    if (warp == 0) {
      // lane owns bins [8*lane, 8*lane + 8)
      uint32_t loc[8], run = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) { loc[k] = hist[lane * 8 + k]; run += loc[k]; }
      uint32_t incl = run;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t excl = incl - run;
      const int64_t kth = sh_kth;
      // the lane whose range holds the kth element picks the bucket
      if ((int64_t)excl < kth && kth <= (int64_t)incl) {
        uint32_t before = excl;
        int bsel = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if ((int64_t)(before + loc[k]) >= kth) { bsel = lane * 8 + k; break; }
          before += loc[k];
        }
        const int64_t rem = kth - before;
        sh_kth = rem;
        sh_prefix = prefix | ((uint64_t)bsel << shift);
        sh_mask = mask | ((uint64_t)0xFFu << shift);
        if ((int64_t)hist[bsel] == rem) sh_done = 1;   // the whole bucket is taken
      }
      if (lane == 31 && (int64_t)incl < kth) {        // fewer eligible slots than needed
        atomicOr(err, kErrSelect);
        sh_done = 2;
      }
    }
    __syncthreads();
  }
  if (sh_done == 2) return;

  // compaction in ascending slot order: eligible and (key & mask) <= prefix
  const uint64_t prefix = sh_prefix, mask = sh_mask;
  int64_t written = 0;
  if (need > 0) {
    for (int64_t base = 0; base < M; base += kSelThreads) {
      const int64_t s = base + tid;
      bool sel = false;
      if (s < M) {
        const int32_t p = ps[s];
        if (p >= 0 && p < lim) {
          const uint64_t key = (recency ? 0ull : (uint64_t)ordered_bits(sc[s]) << 32) | (uint32_t)p;
          sel = (key & mask) <= prefix;
        }
      }
      const unsigned bal = __ballot_sync(0xffffffffu, sel);
      if (lane == 0) warp_tot[warp] = __popc(bal);
      __syncthreads();
      uint32_t off = 0, tot = 0;
      for (int w = 0; w < kSelThreads / 32; ++w) {
        const uint32_t x = warp_tot[w];
        off += (w < warp) ? x : 0;
        tot += x;
      }
      off += __popc(bal & ((1u << lane) - 1u));
      if (sel && written + off < need) out[written + off] = (int32_t)s;
      written += tot;
      __syncthreads();
    }
    if (tid == 0 && written != need) atomicOr(err, kErrSelect);
  }
  // then the empty slots, in order
  for (int64_t i = tid; i < S - need; i += kSelThreads) out[need + i] = (int32_t)(n_valid + i);
}

// ---------------------------------------------------------------------------
// Scatter: one warp per (b, h, chunk token), 16-byte vector copies.
// ---------------------------------------------------------------------------
__global__ void scatter_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                               uint4* __restrict__ kc, uint4* __restrict__ vc,
                               float* __restrict__ scores, int32_t* __restrict__ pos,
                               const int32_t* __restrict__ freed, const float* __restrict__ newscore,
                               int32_t* __restrict__ evicted, int BH, int64_t S, int64_t M,
                               int row_vecs, int64_t t0) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= (int64_t)BH * S) return;
  const int64_t bh = row / S, i = row - bh * S;
  const int32_t slot = freed[bh * S + i];
  if (slot < 0 || slot >= M) return;
  const int64_t src = row * row_vecs;
  const int64_t dst = (bh * M + slot) * row_vecs;
  for (int c = lane; c < row_vecs; c += 32) {
    kc[dst + c] = k[src + c];
    vc[dst + c] = v[src + c];
  }
  if (lane == 0) {
    evicted[bh * S + i] = pos[bh * M + slot];
    pos[bh * M + slot] = (int32_t)(t0 + i);
    scores[bh * M + slot] = newscore[bh * S + i];
  }
}

}  // namespace

cudaError_t launch_score_reduce(unsigned long long* colacc, int64_t acc_stride, float fx_inv,
                                float* scores, float* newscore, int BH, int64_t S, int64_t M,
                                int64_t n_valid, cudaStream_t st) {
  const int threads = 256;
  dim3 grid((unsigned)((n_valid + S + threads - 1) / threads), (unsigned)BH);
  score_reduce_kernel<<<grid, threads, 0, st>>>(colacc, acc_stride, fx_inv, scores, newscore, S, M,
                                                n_valid);
  return cudaGetLastError();
}

cudaError_t launch_select(const float* scores, const int32_t* pos, int BH, int64_t M, int64_t t0,
                          int64_t R, int64_t need, int64_t n_valid, int64_t S, int32_t* freed,
                          int64_t freed_stride, int* err, cudaStream_t st, int recency) {
  select_kernel<<<BH, kSelThreads, 0, st>>>(scores, pos, M, t0, R, need, n_valid, S, freed,
                                            freed_stride, err, recency);
  return cudaGetLastError();
}

cudaError_t launch_scatter(const void* k, const void* v, void* kc, void* vc, float* scores,
                           int32_t* pos, const int32_t* freed, const float* newscore,
                           int32_t* evicted, int BH, int64_t S, int64_t M, int d, int esize,
                           int64_t t0, cudaStream_t st) {
  const int row_vecs = d * esize / 16;
  const int warps = 8;
  const int64_t rows = (int64_t)BH * S;
  const unsigned blocks = (unsigned)((rows + warps - 1) / warps);
  scatter_kernel<<<blocks, warps * 32, 0, st>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint4*>(kc),
      static_cast<uint4*>(vc), scores, pos, freed, newscore, evicted, BH, S, M, row_vecs, t0);
  return cudaGetLastError();
}

}  // namespace h2o
