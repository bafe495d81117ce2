// The step's tail in one launch: score accumulation, masked selection of the
// slots to evict, and the scatter of the chunk's K/V into the freed slots.
//
// "Learning how to Forget: Fine-tuning for Long-Context Sparse Attention",
// §1 Introduction ¶1 (fixed-size cache, slots evicted once full) and ¶4 (H2O:
// the running sum of summed attention weights ranks the slots); Figure 1(c)
// (per-chunk buffer deltas: the evicted slots and the new K/V rows written
// into them).
//
// One thread-block cluster per (b, KV head); CTA `rank` of the cluster owns
// cache slots [rank * per, (rank + 1) * per) and chunk rows
// [rank * per_s, (rank + 1) * per_s).  Phases, separated by cluster barriers:
//   1. add the summed weights (the fixed-point accumulator row the attention
//      kernel filled, read once and cleared) to the scores of its slots, and
//      form each eligible slot's 64-bit key (order-preserving score bits,
//      token position) in shared memory, counting the keys by their first
//      radix digit on the way; the chunk keys' summed weights are the new
//      tokens' initial scores;
//   2. MSD radix select, 11 bits a pass: the bins are spread over the
//      cluster's CTAs (each group of four bins has an owner); every CTA adds
//      its digit counts into the owners' histograms through distributed shared
//      memory, then all CTAs read the merged bins and take the same decision;
//   3. ordered compaction: per-CTA counts are exchanged through rank 0, and
//      each CTA writes its evicted slots at its offset, ascending;
//   4. scatter of the CTA's chunk rows into the freed slots (the rows were
//      read earlier, so mostly stores remain here), recording the position
//      each slot held before: with the freed list, the chunk's buffer delta.
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "h2o_internal.cuh"
#include "sm100.cuh"

// Phase stamps: with -DH2O_STAMPS (see h2o_kv_cache_b200/stamps.py) thread 0 of
// the first kTailStampCtas CTAs records clock64() at the phase boundaries
// (kernel start after the dependency wait, end of phase 1, end of the
// selection, end of the compaction, start and end of the scatter); the
// default build compiles every stamp to nothing.
#ifdef H2O_STAMPS
constexpr int kTailStampCtas = 1024, kTailStampSlots = 16;
__device__ unsigned long long g_h2o_tail_stamps[kTailStampCtas * kTailStampSlots];
#define H2O_TAIL_STAMP(i)                                                          \
  do {                                                                             \
    if (threadIdx.x == 0 && blockIdx.x < kTailStampCtas)                           \
      g_h2o_tail_stamps[blockIdx.x * kTailStampSlots + (i)] = clock64();           \
  } while (0)
// slot 6: the number of radix passes the selection took (a count, not a time);
// slots 7-13: inside the selection's first pass, the compaction and the scatter
#define H2O_TAIL_VALUE(i, v)                                                       \
  do {                                                                             \
    if (threadIdx.x == 0 && blockIdx.x < kTailStampCtas)                           \
      g_h2o_tail_stamps[blockIdx.x * kTailStampSlots + (i)] = (v);                 \
  } while (0)
extern "C" int h2o_tail_stamps_read(unsigned long long* host) {
  return cudaMemcpyFromSymbol(host, g_h2o_tail_stamps, sizeof(g_h2o_tail_stamps)) == cudaSuccess ? 0 : -1;
}
#else
#define H2O_TAIL_STAMP(i) \
  do {                    \
  } while (0)
#define H2O_TAIL_VALUE(i, v) \
  do {                       \
  } while (0)
#endif

namespace h2o {
namespace {

using sm100::smem_u32;

// Bulk (untiled) copy global -> shared of `bytes` (a multiple of 16; both
// addresses 16-byte aligned), completing on the mbarrier `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}
// Waits for the phase of `parity` of a CTA-local mbarrier for at most ~1 s;
// false on a timeout.
__device__ __forceinline__ bool tail_wait(uint32_t bar, uint32_t parity) {
  if (sm100::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = sm100::global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (sm100::mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0 && sm100::global_timer_ns() - t0 > 1000000000ull) return false;
  }
}

constexpr int kTailThreads = 512;
constexpr int kMaxCluster = 16;
constexpr uint64_t kNoKey = ~0ull;   // ineligible slot (a real key has pos < 2^31)
constexpr int kDigitBits = 11;                     // radix digit
constexpr int kBins = 1 << kDigitBits;
constexpr int kBinsPerThread = kBins / kTailThreads;
static_assert(kBinsPerThread == 4, "one 16-byte histogram read per thread");
// chunk rows per warp read ahead on the register path of phase 4: 8 in the
// one-layer kernel; the grouped kernel (many caches per launch) keeps 2 CTAs an
// SM resident instead, which caps it at 64 registers a thread, and its caches
// are large enough for the bulk-copy path
template <int L> constexpr int pre_rows() { return L == 1 ? 8 : 1; }
template <int L> constexpr int min_blocks() { return L == 1 ? 1 : 2; }

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The two halves of cluster_sync(), for work that can overlap the barrier.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of `p` (a shared variable of this CTA) in the CTA of cluster rank `rank`.
__device__ __forceinline__ uint32_t dsmem_addr(const void* p, uint32_t rank) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
__device__ __forceinline__ void dsmem_add(uint32_t addr, uint32_t v) {
  asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t dsmem_ld(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint4 dsmem_ld4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void dsmem_st(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ int32_t ld_relaxed(const int32_t* p) {
  int32_t v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ordered_bits(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum over the block; returns this thread's offset, *total
// gets the block's sum.  Every thread must call it.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t x, uint32_t* warp_sum, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  uint32_t before = 0, all = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
    const uint32_t s = warp_sum[w];
    before += (w < warp) ? s : 0u;
    all += s;
  }
  __syncthreads();   // warp_sum may be reused right after
  *total = all;
  return before + incl - x;
}

// One launch serves a group of L layers of identical sizes: clusters
// [l * BH, (l + 1) * BH) take layer l's (b, KV head) caches.
constexpr int kMaxGroup = 32;
template <int L>
struct TailGroup {
  TailArgs t[L];
  int BH;
  int stage;   // 1: each CTA copies all of its chunk rows into shared memory at the start
};

template <int L>
__global__ void __launch_bounds__(kTailThreads, min_blocks<L>()) tail_kernel(const __grid_constant__ TailGroup<L> grp) {
  constexpr int kPre = pre_rows<L>();
  extern __shared__ __align__(16) unsigned char dyn[];
  uint64_t* keys = reinterpret_cast<uint64_t*>(dyn);                   // [per]
  float* ns = reinterpret_cast<float*>(dyn + (size_t)grp.t[0].per * 8);   // [per_s]
  __shared__ __align__(16) uint32_t hist[3][kBins];   // merged counts of the bins this CTA owns
  __shared__ __align__(16) uint32_t hloc[kBins];      // this CTA's counts of a pass
  __shared__ uint32_t red_sum[kTailThreads / 32];
  __shared__ uint32_t cnt[kMaxCluster];               // rank 0: selected slots per rank
  __shared__ uint32_t warp_sum[kTailThreads / 32];
  __shared__ uint64_t sh_prefix, sh_mask;
  __shared__ int64_t sh_kth;
  __shared__ int sh_state;                            // 0 searching, 1 found, 2 too few
  __shared__ uint32_t sh_off, sh_tot;
  __shared__ __align__(8) uint64_t row_bar[2];        // bulk loads of chunk rows

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nthr = kTailThreads, nwarps = kTailThreads / 32;
  const uint32_t rank = cluster_rank(), cs = cluster_size();
  // a cluster of one CTA needs only the CTA barrier (the cluster barrier's
  // release would also wait for every global store in flight)
  auto csync = [&] {
    if (cs == 1) __syncthreads();
    else cluster_sync();
  };
  const int64_t item = blockIdx.x / cs;                 // (layer, b, KV head)
  const int layer = L == 1 ? 0 : (int)(item / grp.BH);
  const int64_t bh = item - (int64_t)layer * grp.BH;
  const TailArgs& p = grp.t[layer];
  const int64_t M = p.M, S = p.S, nv = p.n_valid, need = p.need;
  const int64_t lo = (int64_t)rank * p.per, hi = lo + p.per < M ? lo + p.per : M;
  const int64_t nloc = hi > lo ? hi - lo : 0;
  const int64_t lo_s = (int64_t)rank * p.per_s, hi_s = lo_s + p.per_s < S ? lo_s + p.per_s : S;

  // the first two passes' histograms and this CTA's counts start at zero; the
  // cluster barrier that makes the zeros visible to the other CTAs' adds is
  // split: arrived at here, waited for after phase 1, which hides its latency
  for (int i = tid; i < 2 * kBins; i += nthr) (&hist[0][0])[i] = 0u;
  for (int i = tid; i < kBins; i += nthr) hloc[i] = 0u;
  if (tid == 0) {
    sh_prefix = 0;
    sh_mask = 0;
    sh_kth = need;
    sh_state = need == 0 ? 1 : 0;
  }
  __syncthreads();
  if (cs > 1) cluster_arrive();
  // everything below reads what the preceding kernel of the stream wrote
  asm volatile("griddepcontrol.wait;" ::: "memory");
  H2O_TAIL_STAMP(0);

  // The CTA's chunk rows reach phase 4 one of three ways.
  //  - Staged (the one-layer kernel when they fit; see below): bulk-copied into
  //    shared memory after phase 1.
  //  - Bulk (the grouped kernel): phase 4 copies them into the keys' shared
  //    memory, free by then, one bulk copy per batch of nb rows (two batches in
  //    flight), and the warps store them to their slots; with two CTAs an SM
  //    and 64 registers a thread it could not keep enough rows in flight in
  //    registers.
  //  - Registers (rows too large to stage): chunk rows i = lo_s + warp +
  //    k * nwarps (k = 0, 1, ...) are this warp's to scatter, the first kPre
  //    read now so that their latency hides behind phases 1-3 (lane c holds
  //    vector c of the row's K vectors followed by its V vectors), then 8 rows
  //    a warp in flight at a time.
  // Measured at 32k/2k (8 caches): phase 4 took 10.2k cycles from registers and
  // 22k through bulk copies in phase 4 for a CTA's 256 rows (clusters of 8),
  // and staged 8.1k for its 205 rows (clusters of 10).
  const int rv = p.row_vecs, vecs2 = 2 * rv;
  const uint32_t row_bytes = (uint32_t)rv * 16u;
  const int64_t n_rows = hi_s > lo_s ? hi_s - lo_s : 0;
  int nb = (int)((int64_t)p.per * 8 / (4 * (int64_t)row_bytes));
  if (nb > 64) nb = 64;
  const bool bulk = L > 1 && nb >= 16 && n_rows > 0;
  // Staged (the one-layer kernel, when the launch sized shared memory for it):
  // the CTA's chunk K rows, then its V rows, are copied into shared memory
  // after the keys by bulk copies of at most 16 KB completing on row_bar[0],
  // issued when phase 1's loads are done (so they do not delay them) and
  // landing during the selection; phase 4 then only stores them to their slots.
  const bool staged = L == 1 && grp.stage != 0 && n_rows > 0;
  const uint32_t stage_off = ((uint32_t)grp.t[0].per * 8u + (uint32_t)grp.t[0].per_s * 4u + 15u) & ~15u;
  if ((bulk || staged) && tid == 0) {
    sm100::mbar_init(smem_u32(&row_bar[0]), 1);
    sm100::mbar_init(smem_u32(&row_bar[1]), 1);
    sm100::fence_mbar_init();
  }
  const bool pre_ok = vecs2 <= 32 && !bulk && !staged;
  const int64_t n_mine = hi_s - lo_s > warp ? (hi_s - lo_s - warp + nwarps - 1) / nwarps : 0;
  uint4 pre[kPre];
  if (pre_ok) {
#pragma unroll
    for (int k = 0; k < kPre; ++k) {
      if (k < n_mine && lane < vecs2) {
        const int64_t src = (bh * S + lo_s + warp + (int64_t)k * nwarps) * rv;
        pre[k] = lane < rv ? __ldg(p.k + src + lane) : __ldg(p.v + src + lane - rv);
      }
    }
  }

  // ---- 1. scores += summed weights (the accumulator words are read and
  // cleared for the next chunk); keys of the eligible slots, and their counts
  // by the selection's first digit (its first pass's histogram); the chunk
  // rows' initial scores.  Four slots a thread per round.
  unsigned long long* acc = p.colacc + bh * p.acc_stride;
  float* sc = p.scores + bh * M;
  int32_t* ps = p.pos + bh * M;
  const int64_t lim = p.t0 - p.R;               // eligible: 0 <= pos < t0 - R
  const bool vec = (M & 3) == 0;                // rows of scores / positions 16-byte aligned
  // Two rounds' loads are issued before either round's stores, so twice the
  // bytes are in flight (the stores could alias the loads as far as the
  // compiler knows, and would otherwise hold back the next round's loads).
  struct Round {
    float sc[4];
    int32_t ps[4];
    unsigned long long av[4];
  };
  auto load_round = [&](int64_t s0, Round& x) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x.sc[e] = 0.f;
      x.ps[e] = -1;
      x.av[e] = 0ull;
    }
    if (s0 >= hi) return;
    if (vec && s0 + 4 <= hi) {
      const float4 f = *reinterpret_cast<const float4*>(sc + s0);
      const int4 q = *reinterpret_cast<const int4*>(ps + s0);
      x.sc[0] = f.x; x.sc[1] = f.y; x.sc[2] = f.z; x.sc[3] = f.w;
      x.ps[0] = q.x; x.ps[1] = q.y; x.ps[2] = q.z; x.ps[3] = q.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (s0 + e < hi) {
          x.sc[e] = sc[s0 + e];
          x.ps[e] = ps[s0 + e];
        }
    }
    if (s0 + 4 <= nv) {                         // acc rows and s0 are multiples of 4 words
      const ulonglong2* a2 = reinterpret_cast<const ulonglong2*>(acc + s0);
      const ulonglong2 x0 = a2[0], x1 = a2[1];
      x.av[0] = x0.x; x.av[1] = x0.y; x.av[2] = x1.x; x.av[3] = x1.y;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (s0 + e < nv) x.av[e] = acc[s0 + e];
    }
  };
  // finish_round leaves the round's keys in x.av (kNoKey past the CTA's slots)
  auto finish_round = [&](int64_t s0, Round& x) {
    if (s0 >= hi) {
#pragma unroll
      for (int e = 0; e < 4; ++e) x.av[e] = kNoKey;
      return;
    }
    if (s0 + 4 <= nv) {
      ulonglong2* a2 = reinterpret_cast<ulonglong2*>(acc + s0);
      a2[0] = make_ulonglong2(0ull, 0ull);
      a2[1] = make_ulonglong2(0ull, 0ull);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (s0 + e < nv) acc[s0 + e] = 0ull;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int64_t s = s0 + e;
      if (s >= hi) {
        x.av[e] = kNoKey;
        continue;
      }
      float v = x.sc[e];
      if (s < nv) v += colsum_value(x.av[e], p.fx_inv);
      x.sc[e] = v;
      const int32_t q = x.ps[e];
      const uint64_t key = (q >= 0 && q < lim)
                               ? (p.recency ? 0ull : (uint64_t)ordered_bits(v) << 32) | (uint32_t)q
                               : kNoKey;
      keys[s - lo] = key;
      x.av[e] = key;
    }
    if (s0 < nv) {
      if (vec && s0 + 4 <= hi) {
        *reinterpret_cast<float4*>(sc + s0) = make_float4(x.sc[0], x.sc[1], x.sc[2], x.sc[3]);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (s0 + e < nv) sc[s0 + e] = x.sc[e];
      }
    }
  };
  // the one-layer kernel loads the thread's first chunk-key word together with
  // its first slots (the grouped kernel has no registers to spare for it)
  const int64_t i_first = L == 1 ? lo_s + tid : hi_s;
  const unsigned long long a_first = i_first < hi_s ? acc[M + i_first] : 0ull;
  // counts of keys by their first digit, a warp's equal digits added at once
  auto count_first_digits = [&](const unsigned long long (&k4)[4]) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bool take = k4[e] != kNoKey;
      const uint32_t digit = (uint32_t)(k4[e] >> (64 - kDigitBits));
      const unsigned act = __ballot_sync(0xffffffffu, take);
      if (take) {
        const unsigned peers = __match_any_sync(act, digit);
        if ((__ffs(peers) - 1) == lane) atomicAdd(&hloc[digit], (uint32_t)__popc(peers));
      }
    }
  };
  for (int64_t base = lo; base < hi; base += 8 * (int64_t)nthr) {   // the same trip count for every thread
    const int64_t s0 = base + 4 * (int64_t)tid, s1 = s0 + 4 * (int64_t)nthr;
    Round ra, rb;
    load_round(s0, ra);
    load_round(s1, rb);
    finish_round(s0, ra);
    finish_round(s1, rb);
    count_first_digits(ra.av);
    count_first_digits(rb.av);
  }
  if (i_first < hi_s) {
    ns[i_first - lo_s] = colsum_value(a_first, p.fx_inv);
    acc[M + i_first] = 0ull;
  }
  for (int64_t i = L == 1 ? i_first + nthr : lo_s + tid; i < hi_s; i += nthr) {
    ns[i - lo_s] = colsum_value(acc[M + i], p.fx_inv);
    acc[M + i] = 0ull;
  }
  if (staged && tid == 0) {
    const uint32_t bar = smem_u32(&row_bar[0]);
    const uint32_t bytes = (uint32_t)n_rows * row_bytes;
    sm100::mbar_arrive_expect_tx(bar, 2u * bytes);
    const uint32_t kdst = smem_u32(dyn) + stage_off;
    const uint32_t vdst = kdst + (uint32_t)p.per_s * row_bytes;
    const unsigned char* ksrc = reinterpret_cast<const unsigned char*>(p.k + (bh * S + lo_s) * rv);
    const unsigned char* vsrc = reinterpret_cast<const unsigned char*>(p.v + (bh * S + lo_s) * rv);
    for (uint32_t o = 0; o < bytes; o += 16384u) {
      const uint32_t n = bytes - o < 16384u ? bytes - o : 16384u;
      bulk_load(kdst + o, ksrc + o, n, bar);
      bulk_load(vdst + o, vsrc + o, n, bar);
    }
  }
  H2O_TAIL_STAMP(1);
  __syncthreads();                  // the CTA's keys and first-digit counts are complete
  if (cs > 1) cluster_wait();       // every CTA's histograms are zero
  H2O_TAIL_STAMP(7);

  // ---- 2. radix select of the need-th smallest key over the cluster,
  // kDigitBits a pass from the top (the last pass takes the 9 bits left)
  // bins [4 t, 4 t + 4) (thread t's) are owned by rank t % cs: the adds and
  // the reads of a pass are spread over the cluster instead of all landing
  // on one CTA's shared memory
  const uint32_t hist_own = dsmem_addr(&hist[0][0], (uint32_t)tid % cs);
  int pass = 0;
  for (int top = 64; top > 0; top -= kDigitBits, ++pass) {
    if (sh_state != 0) break;                   // uniform: every CTA took the same decisions
    const int shift = top > kDigitBits ? top - kDigitBits : 0;
    const uint32_t dmask = (1u << (top - shift)) - 1u;
    const uint64_t prefix = sh_prefix, mask = sh_mask;
    const int64_t kth = sh_kth;
    const uint32_t H = hist_own + (uint32_t)((pass % 3) * kBins * 4);
    // counts of this CTA's keys in shared memory (the first pass's were taken
    // in phase 1), then one remote add per non-empty bin into its owner's
    // histogram
    if (pass > 0) {
      for (int b = tid; b < kBins; b += nthr) hloc[b] = 0u;
      __syncthreads();
      for (int64_t j0 = 0; j0 < nloc; j0 += nthr) {
        const int64_t j = j0 + tid;
        const uint64_t key = j < nloc ? keys[j] : kNoKey;
        const bool take = key != kNoKey && (key & mask) == prefix;
        const uint32_t digit = (uint32_t)(key >> shift) & dmask;
        const unsigned act = __ballot_sync(0xffffffffu, take);
        if (take) {
          const unsigned peers = __match_any_sync(act, digit);
          if ((__ffs(peers) - 1) == lane) atomicAdd(&hloc[digit], (uint32_t)__popc(peers));
        }
      }
      __syncthreads();
    }
    if (pass == 0) H2O_TAIL_STAMP(8);
    {
      const uint4 c4 = *reinterpret_cast<const uint4*>(&hloc[kBinsPerThread * tid]);
      const uint32_t cv[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
      for (int b = 0; b < kBinsPerThread; ++b)
        if (cv[b] != 0u) dsmem_add(H + (uint32_t)(kBinsPerThread * tid + b) * 4u, cv[b]);
    }
    // the histogram of the next pass was last read before the previous barrier
    for (int b = tid; b < kBins; b += nthr) hist[(pass + 1) % 3][b] = 0u;
    csync();
    if (pass == 0) H2O_TAIL_STAMP(9);
    // thread t reads merged bins [kBinsPerThread * t, kBinsPerThread * (t + 1))
    const uint4 h4 = dsmem_ld4(H + (uint32_t)tid * 16u);
    const uint32_t hv[4] = {h4.x, h4.y, h4.z, h4.w};
    const uint32_t sum = (h4.x + h4.y) + (h4.z + h4.w);
    uint32_t total;
    const uint32_t excl = block_excl_scan(sum, warp_sum, &total);
    if ((int64_t)excl < kth && kth <= (int64_t)(excl + sum)) {
      int64_t before = excl;
#pragma unroll
      for (int b = 0; b < kBinsPerThread; ++b) {
        if (before < kth && kth <= before + (int64_t)hv[b]) {
          const int64_t rem = kth - before;
          sh_prefix = prefix | ((uint64_t)(kBinsPerThread * tid + b) << shift);
          sh_mask = mask | ((uint64_t)dmask << shift);
          sh_kth = rem;
          if ((int64_t)hv[b] == rem) sh_state = 1;   // the whole bucket is evicted
        }
        before += hv[b];
      }
    }
    if (tid == 0 && (int64_t)total < kth) sh_state = 2;
    __syncthreads();
    if (pass == 0) H2O_TAIL_STAMP(10);
  }

  H2O_TAIL_STAMP(2);
  H2O_TAIL_VALUE(6, (unsigned long long)pass);
  // ---- 3. evicted slots in ascending order, then the empty slots.  Warp w
  // takes a contiguous run of Q keys (Q a multiple of 32), lane l the keys l,
  // l + 32, ... of it (a warp reads consecutive words: no shared-memory bank
  // conflicts); the warps' counts give each warp its offset in the CTA, and
  // the CTAs' counts, exchanged through rank 0, each CTA's offset.
  const int state = sh_state;
  const uint64_t prefix = sh_prefix, mask = sh_mask;
  const bool do_sel = need > 0 && state == 1;
  auto selected = [&](int64_t j) -> bool {
    const uint64_t key = keys[j];
    return key != kNoKey && (key & mask) <= prefix;
  };
  // When the selection ended after its first pass (or evicts nothing), the
  // CTA's count is already known -- its keys whose first digit is at most the
  // chosen one, from the first pass's counts -- so it is published first and
  // the exchange's cluster barrier overlaps the warps' counts of their runs.
  // (Every CTA took the same decisions: the branch is uniform over the cluster.)
  const bool early = !do_sel || pass == 1;
  const uint32_t cnt0 = dsmem_addr(&cnt[0], 0);
  if (early) {
    uint32_t c = 0;
    if (do_sel) {
      const uint32_t bsel = (uint32_t)(prefix >> (64 - kDigitBits));
      const uint32_t b0 = (uint32_t)(kBinsPerThread * tid);
      const uint4 c4 = *reinterpret_cast<const uint4*>(&hloc[b0]);
      c = (b0 <= bsel ? c4.x : 0u) + (b0 + 1 <= bsel ? c4.y : 0u) + (b0 + 2 <= bsel ? c4.z : 0u) +
          (b0 + 3 <= bsel ? c4.w : 0u);
    }
    c = __reduce_add_sync(0xffffffffu, c);
    if (lane == 0) red_sum[warp] = c;
    __syncthreads();
    if (tid == 0) {
      uint32_t t = 0;
      for (int w = 0; w < nwarps; ++w) t += red_sum[w];
      dsmem_st(cnt0 + rank * 4u, t);
    }
    if (cs > 1) cluster_arrive();
  }
  H2O_TAIL_STAMP(13);
  const int64_t Q = ((nloc + nwarps - 1) / nwarps + 31) & ~(int64_t)31;
  const int64_t w_lo = (int64_t)warp * Q;
  const int64_t w_hi = w_lo + Q < nloc ? w_lo + Q : nloc;
  uint32_t wcnt = 0;
  if (do_sel)
    for (int64_t j0 = w_lo; j0 < w_hi; j0 += 32)
      wcnt += (uint32_t)__popc(__ballot_sync(0xffffffffu, j0 + lane < w_hi && selected(j0 + lane)));
  if (lane == 0) warp_sum[warp] = wcnt;
  __syncthreads();
  uint32_t woff = 0, cta_sel = 0;
  for (int w = 0; w < nwarps; ++w) {
    const uint32_t x = warp_sum[w];
    woff += w < warp ? x : 0u;
    cta_sel += x;
  }
  if (!early) {
    if (tid == 0) dsmem_st(cnt0 + rank * 4u, cta_sel);
    if (cs > 1) cluster_arrive();
  }
  H2O_TAIL_STAMP(11);
  if (cs > 1) cluster_wait();
  else __syncthreads();
  if (warp == 0) {
    const uint32_t x = lane < (int)cs ? dsmem_ld(cnt0 + (uint32_t)lane * 4u) : 0u;
    const uint32_t off = __reduce_add_sync(0xffffffffu, lane < (int)rank ? x : 0u);
    const uint32_t tot = __reduce_add_sync(0xffffffffu, x);
    if (lane == 0) {
      sh_off = off;
      sh_tot = tot;
    }
  }
  __syncthreads();
  const bool sel_ok = need == 0 || (state == 1 && (int64_t)sh_tot == need);
  int32_t* fr = p.freed + bh * S;
  int32_t* ev = p.evicted + bh * S;   // the delta record: the position each filled slot held
  if (do_sel) {
    int64_t base = (int64_t)sh_off + woff;
    for (int64_t j0 = w_lo; j0 < w_hi; j0 += 32) {
      const int64_t j = j0 + lane;
      const bool sel = j < w_hi && selected(j);
      const unsigned bal = __ballot_sync(0xffffffffu, sel);
      if (sel) {
        const int64_t o = base + __popc(bal & ((1u << lane) - 1u));
        if (o < need) {
          fr[o] = (int32_t)(lo + j);
          ev[o] = (int32_t)(uint32_t)keys[j];   // the key's low word is the slot's position
        }
      }
      base += __popc(bal);
    }
  }
  if (rank == 0 && tid == 0 && !sel_ok) atomicOr(p.err, kErrSelect);
  for (int64_t e = (int64_t)rank * nthr + tid; e < S - need; e += (int64_t)cs * nthr) {
    fr[need + e] = (int32_t)(nv + e);
    ev[need + e] = -1;
  }
  H2O_TAIL_STAMP(3);
  csync();   // the freed list is complete; no CTA's shared memory is read remotely any more
  H2O_TAIL_STAMP(4);

  // ---- 4. chunk row i -> slot fr[i]: K and V rows, pos = t0 + i, initial score
  if (staged) {
    // every copy has landed before the CTA goes on, or leaves
    if (!__syncthreads_and(tail_wait(smem_u32(&row_bar[0]), 0u))) {
      if (tid == 0) atomicOr(p.err, kErrTimeout);
      tail_wait(smem_u32(&row_bar[0]), 0u);   // once more (bounded) before the shared memory goes
      return;
    }
    H2O_TAIL_STAMP(12);
    if (!sel_ok) return;
    // a warp per row (rows warp, warp + nwarps, ...): shared memory -> the
    // row's slot, 16 bytes a lane; lane u fetches the slot of the warp's u-th
    // row, so one load latency covers 32 rows
    const uint4* kst = reinterpret_cast<const uint4*>(dyn + stage_off);
    const uint4* vst = kst + (size_t)p.per_s * rv;
    for (int64_t k0 = 0; k0 < n_mine; k0 += 32) {
      const int32_t my_slot = k0 + lane < n_mine ? ld_relaxed(fr + lo_s + warp + (k0 + lane) * nwarps) : -1;
      const int kn = n_mine - k0 < 32 ? (int)(n_mine - k0) : 32;
      for (int u = 0; u < kn; ++u) {
        const int64_t t = warp + (k0 + u) * nwarps;
        const int64_t i = lo_s + t;
        const int32_t slot = __shfl_sync(0xffffffffu, my_slot, u);
        if (slot < 0 || slot >= M) {
          if (lane == 0) atomicOr(p.err, kErrBounds);
          continue;
        }
        const int64_t dst = (bh * M + slot) * rv;
        for (int c = lane; c < vecs2; c += 32) {
          if (c < rv) p.kc[dst + c] = kst[(size_t)t * rv + c];
          else p.vc[dst + c - rv] = vst[(size_t)t * rv + c - rv];
        }
        if (lane == 0) {
          p.pos[bh * M + slot] = (int32_t)(p.t0 + i);
          p.scores[bh * M + slot] = ns[i - lo_s];
        }
      }
    }
#ifdef H2O_STAMPS
    __syncthreads();
    H2O_TAIL_STAMP(5);
#endif
    return;
  }
  if (!sel_ok) return;
  if (bulk) {
    const uint32_t stage = smem_u32(dyn);
    const uint32_t half = 2u * (uint32_t)nb * row_bytes;     // a batch: nb K rows, then nb V rows
    const int n_batches = (int)((n_rows + nb - 1) / nb);
    const uint4* ksrc = p.k + (bh * S + lo_s) * rv;
    const uint4* vsrc = p.v + (bh * S + lo_s) * rv;
    auto issue = [&](int b) {
      const int64_t r0 = (int64_t)b * nb;
      const uint32_t nr = (uint32_t)(n_rows - r0 < nb ? n_rows - r0 : nb);
      const uint32_t dst = stage + (uint32_t)(b & 1) * half;
      const uint32_t bar = smem_u32(&row_bar[b & 1]);
      sm100::mbar_arrive_expect_tx(bar, 2u * nr * row_bytes);
      bulk_load(dst, ksrc + r0 * rv, nr * row_bytes, bar);
      bulk_load(dst + (uint32_t)nb * row_bytes, vsrc + r0 * rv, nr * row_bytes, bar);
    };
    if (tid == 0) issue(0);
    int issued = 1, waited = 0;
    bool ok = true;
    for (int b = 0; b < n_batches; ++b) {
      // the other half was released by the barrier that ended batch b - 1
      if (b + 1 < n_batches) {
        if (tid == 0) issue(b + 1);
        ++issued;
      }
      ok = __syncthreads_and(tail_wait(smem_u32(&row_bar[b & 1]), (uint32_t)(b >> 1) & 1u));
      if (!ok) break;
      ++waited;
      // a warp per row: shared memory -> the row's slot, 16 bytes a lane
      const int64_t r0 = (int64_t)b * nb;
      const int nr = (int)(n_rows - r0 < nb ? n_rows - r0 : nb);
      const uint4* kst = reinterpret_cast<const uint4*>(dyn + (size_t)(b & 1) * half);
      const uint4* vst = kst + (size_t)nb * rv;
      for (int t = warp; t < nr; t += nwarps) {
        const int64_t i = lo_s + r0 + t;
        const int32_t slot = ld_relaxed(fr + i);
        if (slot < 0 || slot >= M) {
          if (lane == 0) atomicOr(p.err, kErrBounds);
          continue;
        }
        const int64_t dst = (bh * M + slot) * rv;
        for (int c = lane; c < vecs2; c += 32) {
          if (c < rv) p.kc[dst + c] = kst[(size_t)t * rv + c];
          else p.vc[dst + c - rv] = vst[(size_t)t * rv + c - rv];
        }
        if (lane == 0) {
          p.pos[bh * M + slot] = (int32_t)(p.t0 + i);
          p.scores[bh * M + slot] = ns[i - lo_s];
        }
      }
      __syncthreads();   // every warp is done reading this half
    }
    if (!ok) {
      // a load did not land within the limit: record it, and let the loads in
      // flight finish (again bounded) before the CTA's shared memory goes
      if (tid == 0) atomicOr(p.err, kErrTimeout);
      for (int b = waited; b < issued; ++b) tail_wait(smem_u32(&row_bar[b & 1]), (uint32_t)(b >> 1) & 1u);
    }
#ifdef H2O_STAMPS
    __syncthreads();
    H2O_TAIL_STAMP(5);
#endif
    return;
  }
  auto finish_row = [&](int64_t i, int32_t slot) {
    if (lane == 0) {
      p.pos[bh * M + slot] = (int32_t)(p.t0 + i);
      p.scores[bh * M + slot] = ns[i - lo_s];
    }
  };
  int64_t k_from = 0;
  if (pre_ok) {
    // lane k fetches the slot of the warp's k-th row
    const int32_t my_slot = lane < n_mine ? ld_relaxed(fr + lo_s + warp + (int64_t)lane * nwarps) : -1;
#pragma unroll
    for (int k = 0; k < kPre; ++k) {
      if (k < n_mine) {
        const int64_t i = lo_s + warp + (int64_t)k * nwarps;
        const int32_t slot = __shfl_sync(0xffffffffu, my_slot, k);
        if (slot < 0 || slot >= M) {
          if (lane == 0) atomicOr(p.err, kErrBounds);
        } else {
          const int64_t dst = (bh * M + slot) * rv;
          if (lane < rv) p.kc[dst + lane] = pre[k];
          else if (lane < vecs2) p.vc[dst + lane - rv] = pre[k];
          finish_row(i, slot);
        }
      }
    }
    k_from = kPre;
  }
  // the rest of the warp's rows, eight at a time: their loads in flight
  // together; a row of more than 32 vectors (fp32, d = 128) in two passes
  for (int64_t k0 = k_from; k0 < n_mine; k0 += 32) {
    const int32_t my_slot = k0 + lane < n_mine ? ld_relaxed(fr + lo_s + warp + (k0 + lane) * nwarps) : -1;
    const int kn = n_mine - k0 < 32 ? (int)(n_mine - k0) : 32;
    for (int jb = 0; jb < kn; jb += 8) {
      for (int hv = 0; 32 * hv < vecs2; ++hv) {
        const int c = lane + 32 * hv;                    // K row then V row
        uint4 buf[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (jb + u < kn && c < vecs2) {
            const int64_t src = (bh * S + lo_s + warp + (k0 + jb + u) * nwarps) * rv;
            buf[u] = c < rv ? __ldg(p.k + src + c) : __ldg(p.v + src + c - rv);
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (jb + u < kn) {
            const int64_t i = lo_s + warp + (k0 + jb + u) * nwarps;
            const int32_t slot = __shfl_sync(0xffffffffu, my_slot, jb + u);
            if (slot < 0 || slot >= M) {
              if (lane == 0 && hv == 0) atomicOr(p.err, kErrBounds);
            } else {
              const int64_t dst = (bh * M + slot) * rv;
              if (c < rv) p.kc[dst + c] = buf[u];
              else if (c < vecs2) p.vc[dst + c - rv] = buf[u];
              if (hv == 0) finish_row(i, slot);
            }
          }
        }
      }
    }
  }
#ifdef H2O_STAMPS
  __syncthreads();   // every warp's rows are stored
  H2O_TAIL_STAMP(5);
#endif
}

size_t tail_smem(int64_t M, int64_t S, int cs, int* per, int* per_s) {
  const int64_t pr = ((M + cs - 1) / cs + 3) & ~(int64_t)3;
  const int64_t prs = (S + cs - 1) / cs;
  *per = (int)pr;
  *per_s = (int)prs;
  return (size_t)pr * 8 + (size_t)prs * 4;
}

constexpr size_t kTailSmemMax = 180 * 1024;   // plus about 41 KB static

// H2O_TAIL_STAGE=0 keeps the one-layer kernel's chunk rows out of shared memory
// (the register path that rows too large to stage take; same results).
bool tail_stage_enabled() {
  const char* s = getenv("H2O_TAIL_STAGE");
  return !(s && s[0] == '0');
}

}  // namespace

int tail_cluster_size(int64_t M, int64_t S, int BH, bool grouped) {
  static_assert(kMaxCluster == 16, "cluster sizes below assume 16");
  // H2O_TAIL_CS=k asks for clusters of k CTAs (used when that size fits and can
  // be scheduled; otherwise the choice below stands)
  const char* fs = getenv("H2O_TAIL_CS");
  const int forced = fs ? atoi(fs) : 0;
  if (cudaFuncSetAttribute(tail_kernel<1>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess ||
      cudaFuncSetAttribute(tail_kernel<kMaxGroup>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  // Many caches in one launch (grouped layers): one CTA a cache when there are
  // at least two waves of them.  The CTAs then need no cluster barriers, and
  // with two CTAs an SM and more caches than CTA slots the launch streams its
  // bytes at the HBM rate instead of waiting on barrier latency.
  if (grouped && forced < 1) {
    int per, per_s;
    const size_t smem = tail_smem(M, S, 1, &per, &per_s);
    int n = 0;
    if (smem <= kTailSmemMax &&
        cudaFuncSetAttribute(tail_kernel<kMaxGroup>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) == cudaSuccess &&
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, tail_kernel<kMaxGroup>, kTailThreads, smem) == cudaSuccess) {
      int dev = 0, sms = 0;
      if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
          n > 0 && BH >= 2 * n * sms)
        return 1;
    }
    cudaGetLastError();
  }
  // otherwise the least work per SM along the critical path: waves of clusters
  // times the share of a cache each CTA takes (1 / cs); on a tie the fewer
  // waves, then the larger cluster
  int best = 0;
  double best_cost = 1e300;
  int64_t best_waves = INT64_MAX;
  for (int cs = kMaxCluster; cs >= 1; --cs) {
    if (cs > 1 && M < 32LL * cs) continue;       // at least 32 slots a CTA
    int per, per_s;
    const size_t smem = tail_smem(M, S, cs, &per, &per_s);
    if (smem > kTailSmemMax) break;               // grows as cs falls: no smaller size fits
    const void* kern = grouped ? reinterpret_cast<const void*>(tail_kernel<kMaxGroup>)
                               : reinterpret_cast<const void*>(tail_kernel<1>);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
      cudaGetLastError();
      break;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(BH * cs));
    cfg.blockDim = dim3(kTailThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)cs;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    if (n < 1) continue;
    if (cs == forced) return cs;
    const int64_t waves = (BH + n - 1) / n;
    const double cost = (double)waves / cs;
    if (cost < best_cost * (1 - 1e-9) || (cost <= best_cost * (1 + 1e-9) && waves < best_waves)) {
      best_cost = cost;
      best_waves = waves;
      best = cs;
    }
  }
  return best;
}

namespace {

template <int L>
cudaError_t launch_tail_t(const TailArgs* a, int n, int BH, int cs, bool pdl, cudaStream_t st) {
  static_assert(sizeof(TailGroup<L>) <= 32000, "kernel parameter space");
  TailGroup<L> g;
  memset(&g, 0, sizeof(g));
  g.BH = BH;
  size_t smem = 0;
  for (int l = 0; l < n; ++l) {
    g.t[l] = a[l];
    smem = tail_smem(a[l].M, a[l].S, cs, &g.t[l].per, &g.t[l].per_s);
  }
  if (smem > kTailSmemMax) return cudaErrorInvalidValue;
  // the one-layer kernel stages each CTA's chunk rows (K and V) in shared
  // memory when they fit
  g.stage = 0;
  if (L == 1 && tail_stage_enabled()) {
    const size_t at = (smem + 15) & ~(size_t)15;
    const size_t rows = 2 * (size_t)g.t[0].per_s * (size_t)a[0].row_vecs * 16;
    if (at + rows <= kTailSmemMax) {
      smem = at + rows;
      g.stage = 1;
    }
  }
  cudaError_t e = cudaFuncSetAttribute(tail_kernel<L>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((int64_t)n * BH * cs));
  cfg.blockDim = dim3(kTailThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = (unsigned)cs;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, tail_kernel<L>, g);
}

}  // namespace

int tail_max_group() { return kMaxGroup; }

cudaError_t launch_tail_group(const TailArgs* a, int n, int BH, int cs, bool pdl, cudaStream_t st) {
  if (cs < 1 || cs > kMaxCluster || n < 1 || n > kMaxGroup)
    return cudaErrorInvalidValue;
  for (int l = 1; l < n; ++l)
    if (a[l].M != a[0].M || a[l].S != a[0].S) return cudaErrorInvalidValue;
  return n == 1 ? launch_tail_t<1>(a, 1, BH, cs, pdl, st) : launch_tail_t<kMaxGroup>(a, n, BH, cs, pdl, st);
}

cudaError_t launch_tail(const TailArgs& a, int BH, int cs, bool pdl, cudaStream_t st) {
  return launch_tail_group(&a, 1, BH, cs, pdl, st);
}

}  // namespace h2o

#ifdef H2O_STAMPS
// The launch floor of the tail's launch shape: a kernel of the same block size,
// cluster size, grid and dynamic shared memory that does nothing but the
// dependency wait (stamps.py times it between CUDA events after a busy kernel).
namespace {
__global__ void __launch_bounds__(h2o::kTailThreads) tail_empty_kernel() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
}  // namespace
extern "C" int h2o_tail_empty_launch(int cs, int grid, int smem, int pdl, void* stream) {
  if (cs < 1 || cs > h2o::kMaxCluster || grid < cs || grid % cs != 0 || smem < 0) return -1;
  if (cudaFuncSetAttribute(tail_empty_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
      cudaFuncSetAttribute(tail_empty_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
    return -1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(h2o::kTailThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = (unsigned)cs;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, tail_empty_kernel) == cudaSuccess ? 0 : -1;
}
#endif
