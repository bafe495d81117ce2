// Tensor-core (tcgen05 / TMEM / TMA) attention with summed attention weights,
// bf16 inputs, head dimension 128.
//
// "Learning how to Forget: Fine-tuning for Long-Context Sparse Attention":
// Abstract (H2O with a dedicated SDPA kernel), FAQ answer 3 (the SDPA kernel
// also returns the summed attention weights), §1 ¶1 (attention over a
// fixed-size cache), §1 ¶3 (GQA).
//
// One CTA owns the same 128 query rows of two query heads A and B that share a
// KV head (256 rows in all), and walks the keys those rows can see -- the
// valid cache slots, then the chunk's keys up to the causal limit -- twice:
//   sweep 1  S_w = Q_w K^T        (per head w: M = 128 queries, N = 256 keys)
//            -> each row's log-sum-exp;
//   sweep 2  S^T = K [Q_A; Q_B]^T (M = 128 keys, N = 256 queries): each
//            softmax thread owns one key, forms its exact probabilities
//            p = exp(s - lse) for its head's 128 queries, sums them (its column
//            sum, no cross-thread reduction) and writes them to shared memory
//            as P^T; then O^T += V^T P^T (M = 128 = d, N = 256 queries), both
//            operands MN-major.  Each key's column sum of each head is added
//            to the (b, KV head)'s fixed-point accumulator row.
// Split keys: a unit of work (two heads' 128 rows) may be shared by a cluster
// of kc CTAs, each taking a contiguous run of its 256-key pairs.  After sweep 1
// every CTA publishes its rows' (max, sum) in shared memory, and each CTA
// combines all of them in rank order into the same log-sum-exp (distributed
// shared memory, remote mbarrier arrivals); after sweep 2 the partial O of
// every CTA is staged in shared memory and rank q adds, in rank order, the
// partials of its 256 / kc rows.  Column sums need no exchange: every key
// belongs to one CTA.  Small chunks (S = 128: two-heads units are few) and
// grids that would leave a partial last wave use kc > 1.
// Exact probabilities mean O needs no rescaling.  Every MMA has N = 256, the
// widest one CTA issues: a key tile takes the fewest MMA instructions and
// commits.
//
// Warp roles (320 threads): warp 0 issues TMA loads (one thread), warp 1
// allocates TMEM and issues the MMAs (one thread), warps 2-5 / 6-9 are two
// softmax warpgroups (thread = TMEM lane).  In sweep 1 both read each head's S
// tile, warpgroup w taking keys [128 w, 128 w + 128) of it, and their (max,
// sum) halves are merged once per unit; in sweep 2 warpgroup w takes head w's
// query columns.  TMEM: sweep 1 holds S_A and S_B (256 columns each); sweep 2
// holds S^T and O^T (256 each).  Every mbarrier wait is bounded; a wait that
// runs out sets the kErrTimeout bit of the device error word and all roles
// exit.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstring>
#include <mutex>

#include "attn_common.cuh"

// Pipeline stamps: with -DH2O_STAMPS (a separate build, see
// h2o_kv_cache_b200/stamps.py) the CTAs of the first wave record clock64() at
// the hand-offs of their first unit -- per 256-key pair of sweep 1 and per
// 128-key tile of sweep 2 -- into a file-scope array that h2o_stamps_read()
// copies out.  The default build compiles every stamp to nothing.
#ifdef H2O_STAMPS
namespace h2o_stamps {
constexpr int kCtas = 148, kSlots = 1200;
}
__device__ unsigned long long g_h2o_stamps[h2o_stamps::kCtas * h2o_stamps::kSlots];
#define H2O_STAMP(i)                                                                     \
  do {                                                                                   \
    if (blockIdx.x < h2o_stamps::kCtas && (i) < h2o_stamps::kSlots)                       \
      g_h2o_stamps[blockIdx.x * h2o_stamps::kSlots + (i)] = clock64();                  \
  } while (0)
extern "C" int h2o_stamps_read(unsigned long long* host) {
  return cudaMemcpyFromSymbol(host, g_h2o_stamps, sizeof(g_h2o_stamps)) == cudaSuccess ? 0 : -1;
}
// every CTA (up to kUnitCtas): its SM, and the global timer at entry and exit
namespace h2o_stamps {
constexpr int kUnitCtas = 16384;
}
__device__ unsigned long long g_h2o_unit_stamps[h2o_stamps::kUnitCtas * 3];
#define H2O_UNIT_STAMP(k, v)                                                   \
  do {                                                                         \
    if (threadIdx.x == 0 && blockIdx.x < h2o_stamps::kUnitCtas)                \
      g_h2o_unit_stamps[blockIdx.x * 3 + (k)] = (v);                           \
  } while (0)
extern "C" int h2o_unit_stamps_read(unsigned long long* host) {
  return cudaMemcpyFromSymbol(host, g_h2o_unit_stamps, sizeof(g_h2o_unit_stamps)) == cudaSuccess ? 0 : -1;
}
#else
#define H2O_STAMP(i) \
  do {               \
  } while (0)
#define H2O_UNIT_STAMP(k, v) \
  do {                       \
  } while (0)
#endif
// stamp slots: [0, 64) producer issues pair u's K tile; [64, 128) MMA warp sees it;
// [128, 256) MMA warp sees head w's S buffer free (128 + 64 w + u); [256, 320) pair
// u's MMAs issued; [320, 448) softmax sees head w's S of pair u; [448, 512) softmax
// ends pair u; sweep 2 tile j: [512, 608) MMA warp starts S^T(j); [608, 704) its
// waits done; [704, 800) O^T(j)'s waits done; [800, 896) softmax sees S^T(j);
// [896, 992) sees P^T free; [992, 1088) has stored P^T(j); 1100 start, 1101 end of
// sweep 1, 1102 end of sweep 2.
enum : int { kStIssueK = 0, kStKFull = 64, kStSEmpty = 128, kStPairIssued = 256, kStSFull = 320,
             kStPairEnd = 448, kStStStart = 512, kStStReady = 608, kStOtReady = 704,
             kStStFull = 800, kStPEmpty = 896, kStPFull = 992, kStStart = 1100,
             kStSweep1End = 1101, kStSweep2End = 1102 };

namespace h2o {
namespace {

using namespace sm100;
using namespace attn;

constexpr int kThreads = 320;
// shared memory: Q (256 rows, K-major: two 32 KB column atoms), then region R
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffR = kOffQ + 2 * kTile;
// sweep 1: two 64 KB slots, each a 256-key K tile (two 32 KB column atoms)
constexpr uint32_t kSlot1 = 2 * kTile;
// sweep 2: three 32 KB slots for K / V tiles, then P^T (128 keys x 256 queries)
constexpr int NS2 = 3;
constexpr uint32_t kOffP = kOffR + NS2 * kTile;
constexpr uint32_t kRBytes = NS2 * kTile + 2 * kTile;   // 160 KB
constexpr uint32_t kOffLse = kOffR + kRBytes;           // negated base-2 lse, [2][128]
constexpr uint32_t kOffBar = kOffLse + 2 * BM * 4;
constexpr int kNumBars = 26;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemUsed = kOffMisc + 16;
// cluster exchange of sweep-1 (max, sum) pairs, [2][128] float2: the part of
// R that neither the sweep-1 slots nor the sweep-2 ring use, and that P^T
// first overwrites only after every CTA of the cluster has read it
constexpr uint32_t kOffX = kOffR + 2 * kSlot1;
static_assert(kOffX >= kOffP && kOffX + 2 * BM * 8 <= kOffR + kRBytes, "exchange inside P^T's tail");
// the two warpgroups' sweep-1 (max, sum) halves, [2][128] float2: right after
// the exchange area, read before any P^T store (a barrier of both warpgroups)
constexpr uint32_t kOffMrg = kOffX + 2 * BM * 8;
static_assert(kOffMrg + 2 * BM * 8 <= kOffR + kRBytes, "merge area inside P^T's tail");
constexpr int kMaxSplit = 8;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;    // slack for 1024-byte alignment
static_assert(2 * kSlot1 <= kRBytes, "sweep-1 slots fit in R");
static_assert(kSmemBytes <= 232448, "shared memory budget");
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitLimitNs = 1000000000ull;     // 1 s per wait
constexpr uint32_t kDescHi = desc_hi_sw128(1024);   // 8 rows of 128 bytes between core-matrix groups

enum { B_Q = 0, B_R1_FULL = 1, B_R1_EMPTY = 3, B_R2_FULL = 5, B_R2_EMPTY = B_R2_FULL + NS2,
       B_S_FULL = B_R2_EMPTY + NS2, B_S_EMPTY = B_S_FULL + 2, B_ST_FULL = B_S_EMPTY + 2,
       B_ST_EMPTY = B_ST_FULL + 1, B_P_FULL = B_ST_EMPTY + 1, B_P_EMPTY = B_P_FULL + 1,
       B_O_FULL = B_P_EMPTY + 1, B_DRAIN = B_O_FULL + 1, B_X_READY = B_DRAIN + 1,
       B_X_READ = B_X_READY + 1,
       B_NEVER = B_X_READ + 1 };   // test hook: nothing ever arrives on it
static_assert(B_NEVER < kNumBars, "barrier count");

struct Params {
  unsigned long long* colacc;      // [B * Hkv][acc_stride] fixed-point summed weights
  int* err;
  void* out;
  int B, Hq, Hkv, G, n_pg, n_rt;
  int units;                       // units of work per layer
  int kc;                          // CTAs (a cluster) per unit of work
  int inject_timeout;              // test hook: make one wait run out
  int64_t S, M, n_valid, acc_stride;
  float scale_log2;   // (1/sqrt(d)) * log2(e)
  float fx_scale;     // 2^fx_shift of the accumulator
};

// A group of L layers that share every size: per layer its five tensor maps
// (q, k, v, cache k, cache v) and its parameters.  One grid covers all the
// layers' units, layer after layer, so a partial last wave is paid once per
// group instead of once per layer.
constexpr int kMaxGroup = 32;
template <int L>
struct Group {
  CUtensorMap maps[L][5];
  Params p[L];
};

template <int L>
__global__ void __launch_bounds__(kThreads, 1)
attn_umma_kernel(const __grid_constant__ Group<L> grp) {
#ifdef H2O_STAMPS
  {
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    H2O_UNIT_STAMP(0, smid);
    H2O_UNIT_STAMP(1, global_timer_ns());
  }
#endif
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  float* nlse = reinterpret_cast<float*>(sbase + kOffLse);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + kOffMisc + 4);
  auto bar = [&](int i) { return base + kOffBar + 8u * (uint32_t)i; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work unit: layer, then (b, h), then row tiles from the last (heaviest), then head pairs
  const int kc = grp.p[0].kc;
  const int rank = (int)(blockIdx.x % (unsigned)kc);        // rank in the cluster
  const int unit_g = (int)(blockIdx.x / (unsigned)kc);
  const int layer = L == 1 ? 0 : unit_g / grp.p[0].units;
  const int unit = unit_g - layer * grp.p[0].units;
  // sizes are the same in every layer of the group (read from layer 0's
  // parameters, which the compiler addresses directly); per layer only the
  // output, the accumulator row and the error word differ
  const Params& p = grp.p[0];
  int* const err = grp.p[layer].err;
  void* const out = grp.p[layer].out;
  unsigned long long* const colacc = grp.p[layer].colacc;
  const CUtensorMap* const tm_q = &grp.maps[layer][0];
  const CUtensorMap* const tm_k = &grp.maps[layer][1];
  const CUtensorMap* const tm_v = &grp.maps[layer][2];
  const CUtensorMap* const tm_kc = &grp.maps[layer][3];
  const CUtensorMap* const tm_vc = &grp.maps[layer][4];
  const int per_bh = p.n_pg * p.n_rt;
  const int bh = unit / per_bh;
  const int k_in = unit - bh * per_bh;
  const int rt = p.n_rt - 1 - k_in / p.n_pg;
  const int pg = k_in % p.n_pg;
  const int b = bh / p.Hkv, h = bh - b * p.Hkv;
  const int gl_a = 2 * pg;                                   // local heads gl_a, gl_a + 1
  const bool has_b = gl_a + 1 < p.G;
  const int64_t i0 = (int64_t)rt * BM;
  const int nct = (int)((p.n_valid + BN - 1) / BN);         // cache tiles
  const int64_t chunk_hi = (i0 + BM < p.S) ? i0 + BM : p.S;   // chunk keys < chunk_hi are visible
  const int nch = (int)((chunk_hi + BN - 1) / BN);
  const int n_all = nct + nch;                                // the unit's 128-key tiles
  const int n1_all = (n_all + 1) >> 1;                        // and its 256-key pairs
  // this CTA's pairs [pr0, pr1), i.e. tiles [t_lo, t_hi); the launch keeps
  // kc <= n1_all, so no CTA is left without keys
  const int pr0 = (int)((int64_t)rank * n1_all / kc), pr1 = (int)((int64_t)(rank + 1) * n1_all / kc);
  const int t_lo = 2 * pr0;
  const int t_hi = 2 * pr1 < n_all ? 2 * pr1 : n_all;
  const int n = t_hi - t_lo;                                  // local 128-key tiles
  const int n1 = pr1 - pr0;                                   // local 256-key tiles

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      uint32_t cnt = 1;
      if (i == B_S_EMPTY || i == B_S_EMPTY + 1) cnt = 256;   // both warpgroups
      if (i == B_ST_EMPTY || i == B_P_FULL) cnt = 256;        // both warpgroups
      if (i == B_X_READY || i == B_X_READ) cnt = (uint32_t)kc;  // one arrival per CTA
      mbar_init(bar(i), cnt);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  if (kc > 1) cluster_sync_all();   // every CTA's barriers exist before remote arrivals
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the cache and the accumulator row may still be in use by the previous kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (threadIdx.x == 0) H2O_STAMP(kStStart);

  // local tile t (128 keys), i.e. the unit's tile t_lo + t: tensor map and row offset
  auto tile_src = [&](int t, bool v, const CUtensorMap*& m, int& y) {
    const int tg = t_lo + t;
    if (tg < nct) {
      m = v ? tm_vc : tm_kc;
      y = tg * BN;
    } else if (tg < t_hi) {
      m = v ? tm_v : tm_k;
      y = (tg - nct) * BN;
    } else {  // past the last tile: a box beyond the chunk's rows reads zeros
      m = v ? tm_v : tm_k;
      y = (int)p.S;
    }
  };

  if (warp == 0) {
    // =========================================================== TMA producer
    if (lane == 0) {
      prefetch_tmap(tm_q);
      prefetch_tmap(tm_k);
      prefetch_tmap(tm_v);
      prefetch_tmap(tm_kc);
      prefetch_tmap(tm_vc);
      // Q: rows of head A then head B, each split into two 64-column atoms
      const int zq = b * p.Hq + h * p.G + gl_a;
      mbar_arrive_expect_tx(bar(B_Q), 2 * kTile);
      for (int hw = 0; hw < 2; ++hw)
        for (int at = 0; at < 2; ++at)
          tma_load_3d(base + kOffQ + at * 2 * kAtom + hw * kAtom, tm_q, bar(B_Q), at * 64, (int)i0,
                      zq + hw);
      bool ok = true;
      int issued1 = 0;                               // sweep-1 tiles whose loads were issued
      // sweep 1: 256-key K tiles into two 64 KB slots
      for (int u = 0; ok && u < n1; ++u) {
        const int s = u & 1;
        ok = mbar_wait(bar(B_R1_EMPTY + s), ((uint32_t)(u >> 1) & 1u) ^ 1u, abort_flag, err,
                       kWaitLimitNs, kErrTimeout);
        if (!ok) break;
        if (u < 64) H2O_STAMP(kStIssueK + u);
        const uint32_t dst = base + kOffR + (uint32_t)s * kSlot1;
        mbar_arrive_expect_tx(bar(B_R1_FULL + s), kSlot1);
        for (int half = 0; half < 2; ++half) {
          const CUtensorMap* m;
          int y;
          tile_src(2 * u + half, false, m, y);
          for (int at = 0; at < 2; ++at)
            tma_load_3d(dst + at * 2 * kAtom + half * kAtom, m, bar(B_R1_FULL + s), at * 64, y, bh);
        }
        issued1 = u + 1;
      }
      // sweep 2 reuses R: wait until every sweep-1 slot has been read
      for (int s = 0; ok && s < 2; ++s) {
        const int fills = (n1 - s + 1) >> 1;
        if (fills > 0)
          ok = mbar_wait(bar(B_R1_EMPTY + s), (uint32_t)(fills - 1) & 1u, abort_flag, err,
                         kWaitLimitNs, kErrTimeout);
      }
      int issued = 0;
      for (int pos = 0; ok && pos < 2 * n; ++pos) {
        const int slot = pos % NS2;
        ok = mbar_wait(bar(B_R2_EMPTY + slot), ((uint32_t)(pos / NS2) & 1u) ^ 1u, abort_flag, err,
                       kWaitLimitNs, kErrTimeout);
        if (!ok) break;
        bool is_v;
        int t;
        if (pos == 0) { is_v = false; t = 0; }
        else if (pos == 2 * n - 1) { is_v = true; t = n - 1; }
        else if (pos & 1) { is_v = false; t = (pos + 1) >> 1; }
        else { is_v = true; t = (pos >> 1) - 1; }
        const CUtensorMap* m;
        int y;
        tile_src(t, is_v, m, y);
        const uint32_t dst = base + kOffR + (uint32_t)slot * kTile;
        mbar_arrive_expect_tx(bar(B_R2_FULL + slot), kTile);
        tma_load_3d(dst, m, bar(B_R2_FULL + slot), 0, y, bh);
        tma_load_3d(dst + kAtom, m, bar(B_R2_FULL + slot), 64, y, bh);
        issued = pos + 1;
      }
      // drain, also after an abort: every load issued has landed before the CTA may exit
      mbar_drain(bar(B_Q), 0, err, kWaitLimitNs, kErrTimeout);
      for (int u = issued1 - 2 < 0 ? 0 : issued1 - 2; u < issued1; ++u)
        mbar_drain(bar(B_R1_FULL + (u & 1)), (uint32_t)(u >> 1) & 1u, err, kWaitLimitNs, kErrTimeout);
      for (int pos = issued - NS2 < 0 ? 0 : issued - NS2; pos < issued; ++pos)
        mbar_drain(bar(B_R2_FULL + pos % NS2), (uint32_t)(pos / NS2) & 1u, err, kWaitLimitNs,
                   kErrTimeout);
    }
  } else if (warp == 1) {
    // =========================================================== MMA issuer
    if (lane == 0) {
      const uint32_t idesc_kk = idesc_bf16(128, 256, 0, 0);   // both operands K-major
      const uint32_t idesc_mn = idesc_bf16(128, 256, 1, 1);   // both operands MN-major
      const uint32_t q_addr = base + kOffQ;
      const uint32_t p_addr = base + kOffP;
      bool ok = mbar_wait(bar(B_Q), 0, abort_flag, err, kWaitLimitNs, kErrTimeout);
      // ---- sweep 1
      for (int u = 0; ok && u < n1; ++u) {
        const int s = u & 1;
        ok = mbar_wait(bar(B_R1_FULL + s), (uint32_t)(u >> 1) & 1u, abort_flag, err, kWaitLimitNs,
                       kErrTimeout);
        if (u < 64) H2O_STAMP(kStKFull + u);
        const uint32_t k_addr = base + kOffR + (uint32_t)s * kSlot1;
        for (int w = 0; ok && w < 2; ++w) {
          ok = mbar_wait(bar(B_S_EMPTY + w), ((uint32_t)u & 1u) ^ 1u, abort_flag, err, kWaitLimitNs,
                         kErrTimeout);
          if (!ok) break;
          if (u < 64) H2O_STAMP(kStSEmpty + 64 * w + u);
          tc_fence_after();
          const uint32_t a0 = desc_lo(q_addr + (uint32_t)w * kAtom, 16), b0 = desc_lo(k_addr, 16);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_bf16(tmem + (uint32_t)w * 256u, a0 + (kmajor_off(kk, 256) >> 4), kDescHi, b0 + (kmajor_off(kk, 256) >> 4),
                      kDescHi, idesc_kk, kk > 0 ? 1u : 0u);
          umma_commit(bar(B_S_FULL + w));
        }
        if (ok) umma_commit(bar(B_R1_EMPTY + s));
        if (u < 64) H2O_STAMP(kStPairIssued + u);
      }
      // ---- sweep 2: S^T(0), S^T(1), O^T(0), S^T(2), O^T(1), ...
      auto issue_st = [&](int j) -> bool {
        if (j < 96) H2O_STAMP(kStStStart + j);
        // TMEM columns 0-255: head A's last sweep-1 S, then S^T(j - 1), must have been read
        bool w_ok = (j == 0)
            ? mbar_wait(bar(B_S_EMPTY + 0), ((uint32_t)n1 & 1u) ^ 1u, abort_flag, err, kWaitLimitNs, kErrTimeout)
            : mbar_wait(bar(B_ST_EMPTY), (uint32_t)(j - 1) & 1u, abort_flag, err, kWaitLimitNs, kErrTimeout);
        const int pos = k_pos(j), slot = pos % NS2;
        if (w_ok)
          w_ok = mbar_wait(bar(B_R2_FULL + slot), (uint32_t)(pos / NS2) & 1u, abort_flag, err,
                           kWaitLimitNs, kErrTimeout);
        if (!w_ok) return false;
        if (j < 96) H2O_STAMP(kStStReady + j);
        tc_fence_after();
        const uint32_t a0 = desc_lo(base + kOffR + (uint32_t)slot * kTile, 16), b0 = desc_lo(q_addr, 16);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_bf16(tmem, a0 + (kmajor_off(kk, 128) >> 4), kDescHi, b0 + (kmajor_off(kk, 256) >> 4), kDescHi, idesc_kk,
                    kk > 0 ? 1u : 0u);
        umma_commit(bar(B_ST_FULL));
        umma_commit(bar(B_R2_EMPTY + slot));
        return true;
      };
      auto issue_ot = [&](int j) -> bool {
        bool w_ok = mbar_wait(bar(B_P_FULL), (uint32_t)j & 1u, abort_flag, err, kWaitLimitNs, kErrTimeout);
        // TMEM columns 256-511: head B's last sweep-1 S must have been read
        if (w_ok && j == 0)
          w_ok = mbar_wait(bar(B_S_EMPTY + 1), ((uint32_t)n1 & 1u) ^ 1u, abort_flag, err,
                           kWaitLimitNs, kErrTimeout);
        const int pos = v_pos(n, j), slot = pos % NS2;
        if (w_ok)
          w_ok = mbar_wait(bar(B_R2_FULL + slot), (uint32_t)(pos / NS2) & 1u, abort_flag, err,
                           kWaitLimitNs, kErrTimeout);
        if (!w_ok) return false;
        if (j < 96) H2O_STAMP(kStOtReady + j);
        tc_fence_after();
        const uint32_t a0 = desc_lo(base + kOffR + (uint32_t)slot * kTile, kAtom), b0 = desc_lo(p_addr, kAtom);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_bf16(tmem + 256u, a0 + (uint32_t)kk * 128u, kDescHi, b0 + (uint32_t)kk * 128u, kDescHi, idesc_mn,
                    (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar(B_P_EMPTY));
        umma_commit(bar(B_R2_EMPTY + slot));
        return true;
      };
      for (int j = 0; ok && j < n; ++j) {
        ok = issue_st(j);
        if (ok && j > 0) ok = issue_ot(j - 1);
      }
      if (ok) ok = issue_ot(n - 1);
      umma_commit(bar(B_O_FULL));
      // every MMA issued has completed before TMEM is released, also after an abort
      umma_commit(bar(B_DRAIN));
      mbar_drain(bar(B_DRAIN), 0, err, kWaitLimitNs, kErrTimeout);
    }
  } else {
    // =========================================================== softmax / epilogue
    const int w = (warp - 2) >> 2;                    // 0: head A, 1: head B
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                 // TMEM lane owned by this thread
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const int64_t S = p.S, M = p.M, nv = p.n_valid;
    const float c = p.scale_log2;
    const bool head_ok = w == 0 || has_b;
    bool ok = true;
    if (p.inject_timeout && w == 0) {
      // test hook: a bounded wait on a barrier nothing completes runs out (1 ms);
      // every role then leaves through its abort path and the step reports it
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_NEVER), 0, abort_flag, err, 1000000ull, kErrTimeout));
    }

    // ----- sweep 1: both warpgroups read each head's S tile, warpgroup w
    // taking keys [128 w, 128 w + 128) of every 256-key tile, so a tile is
    // released after a quarter of the work and the next tile's MMA overlaps
    // the other head's tile.  Thread = query row i0 + r of both heads, with a
    // running (max, sum) of each over its keys; the sum is kept against a
    // reference max that is only raised when a 64-key chunk's max exceeds it
    // by more than 8 (log2 units), so the exponentials of a chunk never wait
    // for that chunk's max.
    const int64_t row_i = i0 + r;
    const int64_t row_lim = (row_i + 1 < S) ? row_i + 1 : S;   // chunk keys < row_lim are seen
    float mh[2] = {-INFINITY, -INFINITY}, lh[2] = {0.f, 0.f};
    auto nvis_of = [&](int t, int half64) -> int {
      const int tg = t_lo + t;
      if (tg >= t_hi) return 0;
      const bool cache = tg < nct;
      const int64_t key0 = (cache ? (int64_t)tg * BN : (int64_t)(tg - nct) * BN) + half64 * 64;
      const int64_t lim = cache ? nv : row_lim;
      return (int)(lim - key0 > 64 ? 64 : (lim - key0 < 0 ? 0 : lim - key0));
    };
    for (int u = 0; ok && u < n1; ++u) {
#pragma unroll
      for (int hw = 0; hw < 2; ++hw) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL + hw), (uint32_t)u & 1u, abort_flag, err,
                                               kWaitLimitNs, kErrTimeout));
        if (threadIdx.x == 64 && u < 64) H2O_STAMP(kStSFull + 64 * hw + u);
        if (!ok) break;
        tc_fence_after();
        const uint32_t s_tmem = lane_base + (uint32_t)hw * 256u + (uint32_t)w * 128u;
#pragma unroll 1
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t v[2][32];
          tmem_ld32(s_tmem + ch * 64, v[0]);
          tmem_ld32(s_tmem + ch * 64 + 32, v[1]);
          tmem_wait_ld();
          if (ch == 1) {
            tc_fence_before();
            mbar_arrive(bar(B_S_EMPTY + hw));
          }
          row_chunk(v, nvis_of(2 * u + w, ch), c, mh[hw], lh[hw]);
        }
      }
      __syncwarp();
      if (threadIdx.x == 64 && u < 64) H2O_STAMP(kStPairEnd + u);
    }
    // warpgroup w finishes head w's rows: it takes the other warpgroup's
    // (max, sum) of them from shared memory.  Every warp passes both barriers
    // whatever its `ok`, so a warp that aborted cannot leave the others waiting.
    float m, l;
    {
      float2* mrg = reinterpret_cast<float2*>(sbase + kOffMrg);
      mrg[(1 - w) * BM + r] = w ? make_float2(mh[0], lh[0]) : make_float2(mh[1], lh[1]);
      named_bar_sync(4, 256);
      const float2 o = mrg[w * BM + r];
      const float m_own = w ? mh[1] : mh[0], l_own = w ? lh[1] : lh[0];
      m = fmaxf(m_own, o.x);
      // an empty half has sum 0 (or NaN when its keys were all masked)
      l = (l_own > 0.f ? l_own * ex2(m_own - m) : 0.f) + (o.y > 0.f ? o.y * ex2(o.x - m) : 0.f);
      named_bar_sync(4, 256);   // both read: P^T may overwrite the area
    }
    // negated base-2 log-sum-exp of each row; -inf zeroes rows past S and a missing head B
    if (kc == 1) {
      nlse[w * BM + r] = (head_ok && row_i < S && l > 0.f) ? -(m + lg2(l)) : -INFINITY;
    } else {
      // publish this CTA's (m, l); once every CTA has, combine them in rank order
      const uint32_t x_own = base + kOffX + (uint32_t)(w * BM + r) * 8u;
      *reinterpret_cast<float2*>(sbase + kOffX + (w * BM + r) * 8) = make_float2(m, l);
      named_bar_sync(3, 256);
      if (threadIdx.x == 64) {
        asm volatile("fence.acq_rel.cluster;" ::: "memory");
        for (int q = 0; q < kc; ++q) mbar_arrive_remote(cluster_map(bar(B_X_READY), (uint32_t)q));
      }
      ok = __all_sync(0xffffffffu, mbar_wait<true>(bar(B_X_READY), 0, abort_flag, err, kWaitLimitNs,
                                                   kErrTimeout));
      float mq[kMaxSplit], lq[kMaxSplit];
      float mx = -INFINITY;
#pragma unroll
      for (int q = 0; q < kMaxSplit; ++q) {
        mq[q] = -INFINITY;
        lq[q] = 0.f;
        if (ok && q < kc) {
          const float2 x = ld_cluster_f2(cluster_map(x_own, (uint32_t)q));
          mq[q] = x.x;
          lq[q] = x.y;
          if (x.y > 0.f) mx = fmaxf(mx, x.x);
        }
      }
      float lsum = 0.f;
#pragma unroll
      for (int q = 0; q < kMaxSplit; ++q)
        if (lq[q] > 0.f) lsum += lq[q] * ex2(mq[q] - mx);
      nlse[w * BM + r] = (head_ok && row_i < S && lsum > 0.f) ? -(mx + lg2(lsum)) : -INFINITY;
      // every CTA's exchange area is overwritten by P^T only after all have read it
      named_bar_sync(3, 256);
      if (threadIdx.x == 64)
        for (int q = 0; q < kc; ++q) mbar_arrive_remote(cluster_map(bar(B_X_READ), (uint32_t)q));
    }
    named_bar_sync(1 + w, 128);
    if (threadIdx.x == 64) H2O_STAMP(kStSweep1End);

    // ----- sweep 2: thread = key (lane r of S^T), the 128 query columns of head w;
    // each warpgroup adds its head's column sum of the key to the accumulator row
    unsigned long long* acc = colacc + (int64_t)bh * p.acc_stride;
    const uint32_t p_row = base + kOffP + (uint32_t)(2 * w) * kAtom + (uint32_t)(r >> 3) * 1024u +
                           (uint32_t)(r & 7) * 128u;
    const float* nl_w = nlse + w * BM;
    const uint32_t st_tmem = lane_base + (uint32_t)w * 128u;
    for (int j = 0; ok && j < n; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_ST_FULL), (uint32_t)j & 1u, abort_flag, err,
                                             kWaitLimitNs, kErrTimeout));
      if (!ok) break;
      if (threadIdx.x == 64 && j < 96) H2O_STAMP(kStStFull + j);
      tc_fence_after();
      const int jg = t_lo + j;
      const bool cache = jg < nct;
      const int64_t key = cache ? (int64_t)jg * BN + r : (int64_t)(jg - nct) * BN + r;
      const bool key_ok = cache ? key < nv : key < S;
      // chunk key `key` is seen by query columns q with i0 + q >= key
      const int qmin = cache ? 0 : (int)(key - i0 > 0 ? key - i0 : 0);
      const bool full = __all_sync(0xffffffffu, key_ok && qmin == 0);
      uint64_t cs4[4] = {0ull, 0ull, 0ull, 0ull};
      // both 64-query halves of this key's P^T row are formed in registers
      // before waiting for the previous tile's O^T MMA to release the buffer,
      // so that MMA overlaps all of this tile's exponentials
      uint32_t pk[32], pk2[32];
      {
        uint32_t v[2][32];
        tmem_ld32(st_tmem, v[0]);
        tmem_ld32(st_tmem + 32, v[1]);
        tmem_wait_ld();
        if (full) key_half<true>(v, nl_w, c, key_ok, qmin, cs4, pk);
        else key_half<false>(v, nl_w, c, key_ok, qmin, cs4, pk);
      }
      {
        uint32_t v[2][32];
        tmem_ld32(st_tmem + 64, v[0]);
        tmem_ld32(st_tmem + 96, v[1]);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar(B_ST_EMPTY));
        if (full) key_half<true>(v, nl_w + 64, c, key_ok, qmin - 64, cs4, pk2);
        else key_half<false>(v, nl_w + 64, c, key_ok, qmin - 64, cs4, pk2);
      }
      if (kc > 1 && j == 0) {   // the cluster is done with the exchange area
        ok = __all_sync(0xffffffffu, mbar_wait<true>(bar(B_X_READ), 0, abort_flag, err,
                                                     kWaitLimitNs, kErrTimeout));
        if (!ok) break;
      }
      // this warpgroup's P^T half of the previous tile has been read by its O^T MMA
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_P_EMPTY), ((uint32_t)j & 1u) ^ 1u, abort_flag,
                                             err, kWaitLimitNs, kErrTimeout));
      if (!ok) break;
      if (threadIdx.x == 64 && j < 96) H2O_STAMP(kStPEmpty + j);
      store_p_half(p_row, r, pk);
      store_p_half(p_row + kAtom, r, pk2);
      fence_async_smem();
      mbar_arrive(bar(B_P_FULL));
      if (threadIdx.x == 64 && j < 96) H2O_STAMP(kStPFull + j);
      // without a head B every probability of warpgroup 1 is 0
      if (key_ok && head_ok) colsum_add(acc + (cache ? key : M + key), cs_total(cs4), p.fx_scale);
    }

    if (threadIdx.x == 64) H2O_STAMP(kStSweep2End);
    // ----- epilogue: O^T (lane = d, columns = queries) -> out rows via shared memory
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_O_FULL), 0, abort_flag, err,
                                                   kWaitLimitNs, kErrTimeout));
    if (kc == 1) {
      // every MMA has completed: R is free; head w's [128 queries x 128 d] goes to R + w * 32 KB.
      // The named barrier is passed by every warp whatever its `ok`, so a warp
      // that aborted cannot leave the others waiting.
      __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(sbase + kOffR + (uint32_t)w * kTile);
      if (ok) {
        tc_fence_after();
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t o[32];
          tmem_ld32(lane_base + 256u + (uint32_t)w * 128u + ch * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) stage[(ch * 32 + k) * D + r] = __float2bfloat16_rn(__uint_as_float(o[k]));
        }
      }
      named_bar_sync(1 + w, 128);
      const int64_t qi = i0 + r;                       // thread r copies query row r
      if (ok && out != nullptr && head_ok && qi < S) {
        const int g = h * p.G + gl_a + w;
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) +
                                              (((int64_t)b * p.Hq + g) * S + qi) * D);
        const uint4* src = reinterpret_cast<const uint4*>(stage + r * D);
#pragma unroll
        for (int k = 0; k < D * 2 / 16; ++k) dst[k] = src[k];
      }
    } else if (ok) {
      tc_fence_after();
      // this CTA's partial O, fp32 [256 queries][128 d], to R (free: every MMA has completed)
      float* stage = reinterpret_cast<float*>(sbase + kOffR);
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t o[32];
        tmem_ld32(lane_base + 256u + (uint32_t)w * 128u + ch * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) stage[(w * BM + ch * 32 + k) * D + r] = __uint_as_float(o[k]);
      }
    }
  }

  if (kc > 1) {
    // every CTA has staged its partial O; rank q sums, in rank order, the rows
    // [q * 256 / kc, (q + 1) * 256 / kc) of all of them and writes them out
    __syncthreads();
    cluster_sync_all();
    if (warp >= 2 && out != nullptr) {
      const int t = threadIdx.x - 64;                 // 0..255
      const int rows = 2 * BM / kc;
      const uint32_t stage0 = base + kOffR;
      for (int it = t; it < rows * (D / 8); it += 256) {
        const int q = rank * rows + it / (D / 8);     // query 0..255: head q / 128, row q % 128
        const int d0 = (it % (D / 8)) * 8;
        const uint32_t off = stage0 + (uint32_t)(q * D + d0) * 4u;
        float4 lo = make_float4(0.f, 0.f, 0.f, 0.f), hi = lo;
        for (int src = 0; src < kc; ++src) {
          const float4 a = ld_cluster_f4(cluster_map(off, (uint32_t)src));
          const float4 c4 = ld_cluster_f4(cluster_map(off + 16u, (uint32_t)src));
          lo.x += a.x; lo.y += a.y; lo.z += a.z; lo.w += a.w;
          hi.x += c4.x; hi.y += c4.y; hi.z += c4.z; hi.w += c4.w;
        }
        const int wq = q / BM;
        const int64_t qi = i0 + (q % BM);
        if ((wq == 0 || has_b) && qi < p.S) {
          const int g = h * p.G + gl_a + wq;
          uint4 v;
          v.x = pack_bf16(lo.x, lo.y);
          v.y = pack_bf16(lo.z, lo.w);
          v.z = pack_bf16(hi.x, hi.y);
          v.w = pack_bf16(hi.z, hi.w);
          *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + (((int64_t)b * p.Hq + g) * p.S + qi) * D + d0) = v;
        }
      }
    }
    cluster_sync_all();   // no CTA leaves while another reads its stage
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  H2O_UNIT_STAMP(2, global_timer_ns());
}

// ---------------------------------------------------------------- host side
// Clusters of kc CTAs that fit on the device at once (1 CTA per SM), per device.
int active_clusters(int kc) {
  static std::mutex mu;
  static int cache[64][kMaxSplit + 1] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 0;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev][kc] == 0) {
    int n = 0;
    if (kc == 1) {
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    } else {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)kc);
      cfg.blockDim = dim3(kThreads);
      cfg.dynamicSmemBytes = kSmemBytes;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = (unsigned)kc;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, attn_umma_kernel<1>, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();
    cache[dev][kc] = n > 0 ? n : -1;
  }
  return cache[dev][kc] > 0 ? cache[dev][kc] : 0;
}

// CTAs per unit of work.  `forced` > 0 asks for that split (capped by what the
// sizes allow); otherwise the split is the one whose waves of clusters take the
// least time, ceil(units / active clusters) / kc, needing a 10% gain over no
// split to pay for the exchanges.  Every CTA keeps at least one 256-key pair.
int split_for(int64_t units, int min_pairs, int forced) {
  int best_kc = 1;
  const int sm = active_clusters(1);
  double best = sm > 0 ? (double)((units + sm - 1) / sm) : 1.0;
  for (int kc = 2; kc <= kMaxSplit; kc *= 2) {
    if (kc > min_pairs) break;
    const int nclu = active_clusters(kc);
    if (nclu < 1) continue;
    if (forced > 0) {
      if (kc <= forced) best_kc = kc;
      continue;
    }
    const double t = (double)((units + nclu - 1) / nclu) / kc;
    if (t < 0.9 * best) {
      best = t;
      best_kc = kc;
    }
  }
  return best_kc;
}

}  // namespace

bool attn_umma_supported(int dtype, int d) { return dtype == kBF16 && d == D; }

namespace {

template <int L>
cudaError_t launch_group(const AttnArgs* a, int n, bool pdl, cudaStream_t st) {
  static_assert(sizeof(Group<L>) <= 32000, "kernel parameter space");
  Group<L> g;
  memset(&g, 0, sizeof(g));
  cudaError_t e = cudaSuccess;
  const int64_t BHq = (int64_t)a[0].B * a[0].Hq, BHkv = (int64_t)a[0].B * a[0].Hkv;
  const int G = a[0].Hq / a[0].Hkv, n_pg = (G + 1) / 2, n_rt = (int)((a[0].S + BM - 1) / BM);
  const int64_t units = BHkv * n_pg * n_rt;
  const int nct = (int)((a[0].n_valid + BN - 1) / BN);
  const int kc = split_for(units * n, (nct + 2) / 2, a[0].split);   // row tile 0 sees nct + 1 tiles
  for (int l = 0; l < n; ++l) {
    const AttnArgs& x = a[l];
    CUtensorMap* m = g.maps[l];
    if ((e = make_map(&m[0], x.q, x.S, BHq)) != cudaSuccess) return e;
    if ((e = make_map(&m[1], x.k, x.S, BHkv)) != cudaSuccess) return e;
    if ((e = make_map(&m[2], x.v, x.S, BHkv)) != cudaSuccess) return e;
    // with an empty cache the cache maps are never read; the chunk's stand in
    const bool has_cache = x.n_valid > 0;
    if ((e = make_map(&m[3], has_cache ? x.kc : x.k, has_cache ? x.M : x.S, BHkv)) != cudaSuccess) return e;
    if ((e = make_map(&m[4], has_cache ? x.vc : x.v, has_cache ? x.M : x.S, BHkv)) != cudaSuccess) return e;
    Params& p = g.p[l];
    p.colacc = x.colacc;
    p.err = x.err;
    p.out = x.out;
    p.B = x.B;
    p.Hq = x.Hq;
    p.Hkv = x.Hkv;
    p.G = G;
    p.n_pg = n_pg;
    p.n_rt = n_rt;
    p.units = (int)units;
    p.kc = kc;
    p.S = x.S;
    p.M = x.M;
    p.n_valid = x.n_valid;
    p.acc_stride = x.acc_stride;
    p.inject_timeout = x.inject_timeout;
    p.scale_log2 = x.scale * 1.4426950408889634f;
    p.fx_scale = fx_scale_of(x.fx_shift);
  }
  e = cudaFuncSetAttribute(attn_umma_kernel<L>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(units * n * kc));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  at[1].id = cudaLaunchAttributeClusterDimension;
  at[1].val.clusterDim.x = (unsigned)kc;
  at[1].val.clusterDim.y = 1;
  at[1].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = kc > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, attn_umma_kernel<L>, g);
}

}  // namespace

int attn_umma_max_group() { return kMaxGroup; }

cudaError_t launch_attn_umma_group(const AttnArgs* a, int n, bool pdl, cudaStream_t st) {
  if (n < 1 || n > kMaxGroup) return cudaErrorInvalidValue;
  for (int l = 0; l < n; ++l) {
    const AttnArgs& x = a[l];
    if (x.d != D) return cudaErrorInvalidValue;
    // one grid serves layers of identical sizes only
    if (x.B != a[0].B || x.Hq != a[0].Hq || x.Hkv != a[0].Hkv || x.S != a[0].S || x.M != a[0].M ||
        x.n_valid != a[0].n_valid || x.fx_shift != a[0].fx_shift || x.split != a[0].split)
      return cudaErrorInvalidValue;
  }
  cudaError_t e = get_encode();
  if (e != cudaSuccess) return e;
  return n == 1 ? launch_group<1>(a, 1, pdl, st) : launch_group<kMaxGroup>(a, n, pdl, st);
}

cudaError_t launch_attn_umma(const AttnArgs& a, bool pdl, cudaStream_t st) {
  return launch_attn_umma_group(&a, 1, pdl, st);
}

}  // namespace h2o
