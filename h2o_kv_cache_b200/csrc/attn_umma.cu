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
// Warp roles (320 threads): warp 0 issues TMA loads, warp 1 allocates TMEM
// and issues the MMAs (one thread), warps 2-9 do the softmax and the epilogue
// as two warpgroups that share the 128 TMEM lanes (thread = lane) and split
// each tile's columns in halves -- twice the warps to hide the latency of the
// exponentials.  TMEM: two 128-column S buffers and a
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
constexpr int NS = 2;              // stages of each of the K and V rings
constexpr int kThreads = 320;      // TMA warp, MMA warp, two softmax warpgroups
constexpr uint32_t kAtom = BM * 64 * 2;          // one [128 x 64] bf16 box: 16 KB
constexpr uint32_t kTile = 2 * kAtom;            // [128 x 128] bf16: 32 KB
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTile;               // K ring: NS tiles
constexpr uint32_t kOffV = kOffK + NS * kTile;          // V ring: NS tiles
constexpr uint32_t kOffP = kOffV + NS * kTile;
constexpr uint32_t kOffLse = kOffP + kTile;
constexpr uint32_t kOffStat = kOffLse + BM * 4;       // row max / sum halves, column-sum hand-over
constexpr uint32_t kOffBar = kOffStat + 6 * BM * 4;
constexpr int kNumBars = 24;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemUsed = kOffMisc + 16;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;    // slack for 1024-byte alignment
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
constexpr uint64_t kWaitLimitNs = 1000000000ull;     // 1 s per wait

// barrier indices
enum { B_Q = 0, B_K_FULL = 1, B_K_EMPTY = B_K_FULL + NS, B_V_FULL = B_K_EMPTY + NS,
       B_V_EMPTY = B_V_FULL + NS, B_S_FULL = B_V_EMPTY + NS,
       B_S_EMPTY = B_S_FULL + 2, B_P_FULL = B_S_EMPTY + 2, B_P_EMPTY = B_P_FULL + 1,
       B_O_FULL = B_P_EMPTY + 1, B_DRAIN = B_O_FULL + 1, B_CS_FULL = B_DRAIN + 1,
       B_CS_EMPTY = B_CS_FULL + 2 };
static_assert(B_CS_EMPTY + 1 < kNumBars, "barrier count");

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
    // S buffers and P are released / filled by both softmax warpgroups (256
    // arrivals); the column-sum hand-over by one (128); the rest by one thread
    for (int i = 0; i < kNumBars; ++i) {
      uint32_t cnt = 1;
      if (i == B_S_EMPTY || i == B_S_EMPTY + 1 || i == B_P_FULL) cnt = 256;
      if (i >= B_CS_FULL && i < B_CS_EMPTY + 2) cnt = 128;
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
      // Loads in the order the MMAs consume them.  K ring: sweep 1's tiles, then
      // sweep 2's; each K stage is freed as soon as its S / S^T MMA is done.  V
      // ring (sweep 2 only): freed when its PV MMA is done.  Sweep 2 order:
      // K0, K1, V0, K2, V1, ... so K(j+1) is never queued behind V(j).
      int k_issued = 0, v_issued = 0;
      auto load_k = [&](int kit) -> bool {
        const int stage = kit % NS;
        if (!mbar_wait(bar(B_K_EMPTY + stage), ((uint32_t)(kit / NS) & 1u) ^ 1u, abort_flag, p.err,
                       kWaitLimitNs, kErrTimeout))
          return false;
        const int t = kit < n ? kit : kit - n;
        const bool cache = t < nct;
        const CUtensorMap* mk = cache ? &tm_kc : &tm_k;
        const int y = cache ? t * BN : (t - nct) * BN;
        const uint32_t dst = base + kOffK + (uint32_t)stage * kTile;
        mbar_arrive_expect_tx(bar(B_K_FULL + stage), kTile);
        tma_load_3d(dst, mk, bar(B_K_FULL + stage), 0, y, bh);
        tma_load_3d(dst + kAtom, mk, bar(B_K_FULL + stage), 64, y, bh);
        k_issued = kit + 1;
        return true;
      };
      auto load_v = [&](int j) -> bool {
        const int stage = j % NS;
        if (!mbar_wait(bar(B_V_EMPTY + stage), ((uint32_t)(j / NS) & 1u) ^ 1u, abort_flag, p.err,
                       kWaitLimitNs, kErrTimeout))
          return false;
        const bool cache = j < nct;
        const CUtensorMap* mv = cache ? &tm_vc : &tm_v;
        const int y = cache ? j * BN : (j - nct) * BN;
        const uint32_t dst = base + kOffV + (uint32_t)stage * kTile;
        mbar_arrive_expect_tx(bar(B_V_FULL + stage), kTile);
        tma_load_3d(dst, mv, bar(B_V_FULL + stage), 0, y, bh);
        tma_load_3d(dst + kAtom, mv, bar(B_V_FULL + stage), 64, y, bh);
        v_issued = j + 1;
        return true;
      };
      bool ok = true;
      for (int kit = 0; ok && kit <= n; ++kit) ok = load_k(kit);      // sweep 1, then K0 of sweep 2
      for (int j = 0; ok && j < n; ++j) {
        if (j + 1 < n) ok = load_k(n + j + 1);
        if (ok) ok = load_v(j);
      }
      // drain: the last loads of each ring have landed before the CTA may exit
      for (int it = k_issued - NS < 0 ? 0 : k_issued - NS; it < k_issued; ++it)
        mbar_wait(bar(B_K_FULL + it % NS), (uint32_t)(it / NS) & 1u, abort_flag, p.err,
                  kWaitLimitNs, kErrTimeout);
      for (int it = v_issued - NS < 0 ? 0 : v_issued - NS; it < v_issued; ++it)
        mbar_wait(bar(B_V_FULL + it % NS), (uint32_t)(it / NS) & 1u, abort_flag, p.err,
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
        if (!mbar_wait(bar(B_K_FULL + stage), (uint32_t)(it / NS) & 1u, abort_flag, p.err,
                       kWaitLimitNs, kErrTimeout))
          return false;
        if (!mbar_wait(bar(B_S_EMPTY + sb), ((uint32_t)(it >> 1) & 1u) ^ 1u, abort_flag, p.err,
                       kWaitLimitNs, kErrTimeout))
          return false;
        tc_fence_after();
        const uint32_t k_addr = base + kOffK + (uint32_t)stage * kTile;
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
        umma_commit(bar(B_K_EMPTY + stage));
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
        const int stage = j % NS;
        if (!mbar_wait(bar(B_V_FULL + stage), (uint32_t)(j / NS) & 1u, abort_flag, p.err,
                       kWaitLimitNs, kErrTimeout)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t v_addr = base + kOffV + (uint32_t)stage * kTile;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t dp = smem_desc_sw128(p_addr + (uint32_t)kk * 2048u, kAtom, 1024);
          const uint64_t dv = smem_desc_sw128(v_addr + (uint32_t)kk * 2048u, kAtom, 1024);
          umma_bf16(tmem + kColO, dp, dv, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar(B_P_EMPTY));
        umma_commit(bar(B_V_EMPTY + stage));
      }
      umma_commit(bar(B_O_FULL));
      // every MMA issued has completed before TMEM is released
      umma_commit(bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0, abort_flag, p.err, kWaitLimitNs, kErrTimeout);
    }
  } else {
    // =========================================================== softmax / epilogue
    // Two warpgroups share every TMEM lane: warpgroup hc (0: warps 2-5, 1: warps
    // 6-9) takes columns [64 hc, 64 hc + 64) of each S / S^T / O tile.
    const int hc = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                 // TMEM lane owned by this thread
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)hc * 64u;
    const int64_t S = p.S, M = p.M, nv = p.n_valid;
    const float c = p.scale_log2;
    float* sm_m = reinterpret_cast<float*>(sbase + kOffStat);        // [2][128]
    float* sm_l = sm_m + 2 * BM;                                      // [2][128]
    float* cs_buf = sm_l + 2 * BM;                                    // [2][128]
    bool ok = true;

    // ----- sweep 1: thread = query row i0 + r, keys of its column half
    const int64_t row_i = i0 + r;
    float m = -INFINITY, l = 0.f;
    for (int it = 0; ok && it < n; ++it) {
      const int sb = it & 1;
      // tcgen05.ld is warp-collective: the whole warp proceeds or stops together
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL + sb), (uint32_t)(it >> 1) & 1u,
                                             abort_flag, p.err, kWaitLimitNs, kErrTimeout));
      if (!ok) break;
      tc_fence_after();
      uint32_t v[2][32];
      tmem_ld32(lane_base + (uint32_t)sb * 128u, v[0]);
      tmem_ld32(lane_base + (uint32_t)sb * 128u + 32u, v[1]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(B_S_EMPTY + sb));
      const bool cache = it < nct;
      const int64_t key0 = (cache ? (int64_t)it * BN : (int64_t)(it - nct) * BN) + hc * 64;
      // keys visible to this row: cache slots < n_valid; chunk keys <= row_i (and < S)
      const int64_t lim = cache ? nv : ((row_i + 1 < S) ? row_i + 1 : S);
      const int nvis = (int)(lim - key0 > 64 ? 64 : (lim - key0 < 0 ? 0 : lim - key0));
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (nvis == 64) {
#pragma unroll
        for (int k = 0; k < 64; ++k) {
          const float x = __uint_as_float(v[k >> 5][k & 31]) * c;
          v[k >> 5][k & 31] = __float_as_uint(x);
          mx4[k & 3] = fmaxf(mx4[k & 3], x);
        }
      } else {
#pragma unroll
        for (int k = 0; k < 64; ++k) {
          const float x = k < nvis ? __uint_as_float(v[k >> 5][k & 31]) * c : -INFINITY;
          v[k >> 5][k & 31] = __float_as_uint(x);
          mx4[k & 3] = fmaxf(mx4[k & 3], x);
        }
      }
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      if (mx > -INFINITY) {
        const float mn = fmaxf(m, mx);
        float s8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < 64; ++k) s8[k & 7] += ex2(__uint_as_float(v[k >> 5][k & 31]) - mn);
        const float sum = ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
        l = (m == -INFINITY ? 0.f : l * ex2(m - mn)) + sum;
        m = mn;
      }
      __syncwarp();
    }
    // combine the two column halves of each row into its log-sum-exp (base 2)
    sm_m[hc * BM + r] = m;
    sm_l[hc * BM + r] = l;
    named_bar_sync(1, 256);
    if (hc == 0) {
      const float ma = sm_m[r], mb = sm_m[BM + r];
      const float la = sm_l[r], lb = sm_l[BM + r];
      const float mm = fmaxf(ma, mb);
      const float ll = (ma == -INFINITY ? 0.f : la * ex2(ma - mm)) + (mb == -INFINITY ? 0.f : lb * ex2(mb - mm));
      // stored negated: sweep 2 forms s * c - lse with one FFMA; -inf zeroes invalid rows
      lse2[r] = (row_i < S && ll > 0.f) ? -(mm + lg2(ll)) : -INFINITY;
    }
    named_bar_sync(1, 256);
    float nl[64];
#pragma unroll
    for (int k = 0; k < 64; k += 4) {
      const float4 t4 = *reinterpret_cast<const float4*>(lse2 + hc * 64 + k);
      nl[k] = t4.x; nl[k + 1] = t4.y; nl[k + 2] = t4.z; nl[k + 3] = t4.w;
    }

    // ----- sweep 2: thread = key (lane r of the S^T tile), query columns of its half
    float* part = p.partials + ((int64_t)bh * (p.G * p.n_rt) + (gl * p.n_rt + rt)) * (M + S);
    const uint32_t p_row = base + kOffP + (uint32_t)hc * kAtom + (uint32_t)(r >> 3) * 1024u +
                           (uint32_t)(r & 7) * 128u;
    for (int j = 0; ok && j < n; ++j) {
      const int it = n + j;
      const int sb = it & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_S_FULL + sb), (uint32_t)(it >> 1) & 1u,
                                             abort_flag, p.err, kWaitLimitNs, kErrTimeout));
      if (!ok) break;
      tc_fence_after();
      uint32_t v[2][32];
      tmem_ld32(lane_base + (uint32_t)sb * 128u, v[0]);
      tmem_ld32(lane_base + (uint32_t)sb * 128u + 32u, v[1]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(B_S_EMPTY + sb));
      const bool cache = j < nct;
      const int64_t key = cache ? (int64_t)j * BN + r : (int64_t)(j - nct) * BN + r;
      const bool key_ok = cache ? key < nv : key < S;
      // chunk key `key` is seen by query columns q with i0 + q >= key
      const int qmin = (cache ? 0 : (int)(key - i0 > 0 ? key - i0 : 0)) - hc * 64;
      float cs8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      uint32_t pk[32];
      if (key_ok && qmin <= 0) {
#pragma unroll
        for (int k = 0; k < 64; k += 2) {
          const float e0 = ex2(fmaf(__uint_as_float(v[k >> 5][k & 31]), c, nl[k]));
          const float e1 = ex2(fmaf(__uint_as_float(v[k >> 5][(k + 1) & 31]), c, nl[k + 1]));
          cs8[k & 7] += e0;
          cs8[(k + 1) & 7] += e1;
          pk[k >> 1] = pack_bf16(e0, e1);
        }
      } else {
#pragma unroll
        for (int k = 0; k < 64; k += 2) {
          float e0 = ex2(fmaf(__uint_as_float(v[k >> 5][k & 31]), c, nl[k]));
          float e1 = ex2(fmaf(__uint_as_float(v[k >> 5][(k + 1) & 31]), c, nl[k + 1]));
          e0 = (key_ok && k >= qmin) ? e0 : 0.f;
          e1 = (key_ok && k + 1 >= qmin) ? e1 : 0.f;
          cs8[k & 7] += e0;
          cs8[(k + 1) & 7] += e1;
          pk[k >> 1] = pack_bf16(e0, e1);
        }
      }
      float cs = ((cs8[0] + cs8[1]) + (cs8[2] + cs8[3])) + ((cs8[4] + cs8[5]) + (cs8[6] + cs8[7]));
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_P_EMPTY), ((uint32_t)j & 1u) ^ 1u, abort_flag,
                                             p.err, kWaitLimitNs, kErrTimeout));
      if (!ok) break;
      // P^T row r (key) -> MN-major P tile, query block hc, 16-byte chunks
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        const uint32_t addr = p_row + (((uint32_t)c8 ^ (uint32_t)(r & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[c8 * 4]),
                     "r"(pk[c8 * 4 + 1]), "r"(pk[c8 * 4 + 2]), "r"(pk[c8 * 4 + 3])
                     : "memory");
      }
      fence_async_smem();
      mbar_arrive(bar(B_P_FULL));
      // the key's column sum over all 128 queries: warpgroup 1 hands its half over
      const int cb = j & 1;
      const uint32_t cph = (uint32_t)(j >> 1) & 1u;
      if (hc == 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(B_CS_EMPTY + cb), cph ^ 1u, abort_flag, p.err,
                                               kWaitLimitNs, kErrTimeout));
        if (!ok) break;
        cs_buf[cb * BM + r] = cs;
        mbar_arrive(bar(B_CS_FULL + cb));
      } else {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(B_CS_FULL + cb), cph, abort_flag, p.err,
                                               kWaitLimitNs, kErrTimeout));
        if (!ok) break;
        cs += cs_buf[cb * BM + r];
        mbar_arrive(bar(B_CS_EMPTY + cb));
        if (key_ok) part[cache ? key : M + key] = cs;
      }
    }

    // ----- epilogue: thread = query row i0 + r, output columns of its half
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_O_FULL), 0, abort_flag, p.err,
                                                   kWaitLimitNs, kErrTimeout));
    if (ok) {
      tc_fence_after();
      uint32_t o[2][32];
      tmem_ld32(lane_base + kColO, o[0]);
      tmem_ld32(lane_base + kColO + 32u, o[1]);
      tmem_wait_ld();
      if (p.out != nullptr && row_i < S) {
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) +
                              (((int64_t)b * p.Hq + g) * S + row_i) * D + hc * 64;
#pragma unroll
        for (int k = 0; k < 64; k += 8) {
          uint4 w;
          w.x = pack_bf16(__uint_as_float(o[k >> 5][k & 31]), __uint_as_float(o[k >> 5][(k + 1) & 31]));
          w.y = pack_bf16(__uint_as_float(o[k >> 5][(k + 2) & 31]), __uint_as_float(o[k >> 5][(k + 3) & 31]));
          w.z = pack_bf16(__uint_as_float(o[k >> 5][(k + 4) & 31]), __uint_as_float(o[k >> 5][(k + 5) & 31]));
          w.w = pack_bf16(__uint_as_float(o[k >> 5][(k + 6) & 31]), __uint_as_float(o[k >> 5][(k + 7) & 31]));
          *reinterpret_cast<uint4*>(orow + k) = w;
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
