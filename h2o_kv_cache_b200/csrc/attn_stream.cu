// Tensor-core attention with summed weights as two persistent kernels over a
// balanced split of the work ("stream-K"), bf16, head dimension 128.
//
// "Learning how to Forget: Fine-tuning for Long-Context Sparse Attention":
// Abstract and FAQ answer 3 (an SDPA kernel that also returns the summed
// attention weights), §1 ¶1 (a fixed-size cache), §1 ¶3 (GQA).
//
// A unit of work is the 128 rows of two query heads (as in attn_umma.cu) and
// its keys, counted in 256-key pairs.  Units differ in size (the causal part
// of the chunk), and 128 or 256 of them on 148 SMs leave SMs idle.  Here the
// units are taken in rounds of whole KV heads, as many heads a round as keep
// their K and V within half of L2 (every CTA works on the same few heads at a
// time, so the second sweep's K and V come from L2); the pairs of a round's
// units form one sequence that is cut into n_cta equal runs, and CTA i takes
// run i of every round: the end of one unit, whole units, and the start of
// another.  Each part of a unit in one CTA is a "piece".
//   kernel A (sweep 1): per piece, S = Q K^T and each row's running (max, sum)
//            over the piece's keys -> global workspace [unit][piece][row];
//   kernel B (sweep 2): per piece, the unit's log-sum-exp from its pieces'
//            (max, sum), in piece order; S^T = K Q^T, exact p, column sums
//            (each key is in one piece: written directly), O^T += V^T P^T.  A
//            unit in one piece writes its output; otherwise each piece writes
//            its fp32 partial O and the last piece to finish (an atomic count
//            per unit) adds all of them in piece order and writes the output.
// No CTA waits on another.  Both kernels use the pipelines of attn_umma.cu
// (TMA producer warp, MMA warp), run back to back over the CTA's pieces, with
// four softmax warpgroups: in kernel A each takes a quarter of every 256-key
// tile's keys for both heads (the four (max, sum) are merged per piece); in
// kernel B each takes 64 query columns of S^T, which is two 128-column
// buffers, one per head, and adds its column sums to the accumulator row.
// Every mbarrier wait is bounded.
#include <cstdio>
#include <vector>

#include "attn_common.cuh"

namespace h2o {
namespace {

using namespace sm100;
using namespace attn;

constexpr int kWg = 4;                           // softmax warpgroups (both kernels)
constexpr int kSoft = 128 * kWg;                 // softmax threads
constexpr int kThreads = 64 + kSoft;             // + TMA producer warp + MMA warp
constexpr int kMaxPieces = 8;                    // per CTA (the host checks)
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per wait
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kDescHi = desc_hi_sw128(1024);   // 8 rows of 128 bytes between core-matrix groups

// kernel A shared memory: Q, two 64 KB slots of 256 keys
constexpr uint32_t kA_OffQ = 0;
constexpr uint32_t kA_OffK = 2 * kTile;
constexpr uint32_t kA_Slot = 2 * kTile;
// the softmax warpgroups' (max, sum) over their keys of a piece's rows,
// [warpgroup][head][128] float2
constexpr uint32_t kA_OffMrg = kA_OffK + 2 * kA_Slot;
constexpr uint32_t kA_OffBar = kA_OffMrg + kWg * 2 * BM * 8;
enum { A_Q = 0, A_Q_EMPTY, A_K_FULL, A_K_EMPTY = A_K_FULL + 2, A_S_FULL = A_K_EMPTY + 2,
       A_S_EMPTY = A_S_FULL + 2, A_DRAIN = A_S_EMPTY + 2, A_NUM = A_DRAIN + 1 };

// kernel B shared memory: Q, a ring of three 32 KB K / V slots, P^T (64 KB),
// the rows' negated log-sum-exp
constexpr int NS2 = 3;
constexpr uint32_t kB_OffQ = 0;
constexpr uint32_t kB_OffR = 2 * kTile;
constexpr uint32_t kB_OffP = kB_OffR + NS2 * kTile;
constexpr uint32_t kB_OffLse = kB_OffP + 2 * kTile;
constexpr uint32_t kB_OffBar = kB_OffLse + 2 * BM * 4;
// S^T is two buffers of 128 columns, one per head (TMEM columns 0-127: head
// A's queries, 128-255: head B's), each with its own full / empty barriers,
// so the softmax reads one head's tile while the other head's MMA runs
enum { B_Q = 0, B_Q_EMPTY, B_R_FULL, B_R_EMPTY = B_R_FULL + NS2, B_ST_FULL = B_R_EMPTY + NS2,
       B_ST_EMPTY = B_ST_FULL + 2, B_P_FULL = B_ST_EMPTY + 2, B_P_EMPTY, B_O_FULL, B_O_EMPTY, B_DRAIN,
       B_NEVER,   // test hook: nothing ever arrives on it
       B_NUM };

// after the barriers: TMEM address, abort flag, the CTA's pieces
struct Piece {
  int u;       // unit
  int a, c;    // the unit's pairs [a, c)
  int k, np;   // piece index within the unit, and the unit's number of pieces
};
constexpr uint32_t kMiscBytes = 16 + kMaxPieces * sizeof(Piece) + 16;
constexpr uint32_t kA_SmemBytes = kA_OffBar + A_NUM * 8 + kMiscBytes + 1024;
constexpr uint32_t kB_SmemBytes = kB_OffBar + B_NUM * 8 + kMiscBytes + 1024;
static_assert(kA_SmemBytes <= 232448 && kB_SmemBytes <= 232448, "shared memory budget");

struct SParams {
  unsigned long long* colacc;   // fixed-point summed weights, [BHkv][acc_stride]
  int* err;
  void* out;            // [B, Hq, S, D] bf16, or null
  float2* ws_ml;        // [units][maxp][2 * BM]: a piece's rows' (max, sum), base 2
  float* ws_o;          // [units][maxp][2 * BM][D]: a piece's partial O (split units)
  int* count;           // [units]: pieces of the unit done with sweep 2
  int B, Hq, Hkv, G, n_pg, n_rt, maxp;
  int inject_timeout;   // test hook: one wait of kernel B runs out
  int64_t S, M, n_valid, acc_stride;
  int heads_per_round;  // (b, KV head) caches per round
  float scale_log2;
  float fx_scale;       // 2^fx_shift of the accumulator
};

// ---- units: u = (bh * n_pg + pg) * n_rt + rt
struct UnitGeo {
  int bh, b, h, pg, rt, gl_a;
  bool has_b;
  int64_t i0;
  int nct, n_all;       // cache tiles, all 128-key tiles
};
__device__ __forceinline__ UnitGeo unit_geo(const SParams& p, int u) {
  UnitGeo g;
  g.rt = u % p.n_rt;
  const int t = u / p.n_rt;
  g.pg = t % p.n_pg;
  g.bh = t / p.n_pg;
  g.b = g.bh / p.Hkv;
  g.h = g.bh - g.b * p.Hkv;
  g.gl_a = 2 * g.pg;
  g.has_b = g.gl_a + 1 < p.G;
  g.i0 = (int64_t)g.rt * BM;
  g.nct = (int)((p.n_valid + BN - 1) / BN);
  const int64_t chunk_hi = (g.i0 + BM < p.S) ? g.i0 + BM : p.S;
  g.n_all = g.nct + (int)((chunk_hi + BN - 1) / BN);
  return g;
}
__device__ __forceinline__ int unit_pairs(const SParams& p, int u) {
  return (unit_geo(p, u).n_all + 1) >> 1;
}
// CTA whose run holds pair g of a round of P pairs: runs start at floor(i * P / n_cta)
__host__ __device__ __forceinline__ int cta_of(int64_t g, int64_t P, int n_cta) {
  return (int)(((g + 1) * n_cta + P - 1) / P) - 1;
}

// Thread 0: this CTA's pieces into shared memory, round after round; returns
// their number (-1 if more than kMaxPieces).
__device__ int build_pieces(const SParams& p, Piece* pc) {
  const int n_cta = gridDim.x;
  const int BH = p.B * p.Hkv, per_head = p.n_pg * p.n_rt;
  int n = 0;
  for (int h0 = 0; h0 < BH; h0 += p.heads_per_round) {
    const int u_lo = h0 * per_head;
    const int u_hi = (h0 + p.heads_per_round < BH ? h0 + p.heads_per_round : BH) * per_head;
    int64_t P = 0;
    for (int u = u_lo; u < u_hi; ++u) P += unit_pairs(p, u);
    const int64_t lo = (int64_t)blockIdx.x * P / n_cta, hi = (int64_t)(blockIdx.x + 1) * P / n_cta;
    int64_t g0 = 0;   // first pair of unit u within the round
    for (int u = u_lo; u < u_hi && g0 < hi; ++u) {
      const int q = unit_pairs(p, u);
      const int64_t g1 = g0 + q;
      if (g1 > lo) {
        if (n == kMaxPieces) return -1;
        Piece& x = pc[n++];
        x.u = u;
        x.a = (int)((lo > g0 ? lo : g0) - g0);
        x.c = (int)((hi < g1 ? hi : g1) - g0);
        const int first = cta_of(g0, P, n_cta), last = cta_of(g1 - 1, P, n_cta);
        x.k = (int)blockIdx.x - first;
        x.np = last - first + 1;
      }
      g0 = g1;
    }
  }
  return n;
}


// ------------------------------------------------------------------ kernel A
__global__ void __launch_bounds__(kThreads, 1)
lse_stream_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_kc, const SParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  uint8_t* misc = sbase + kA_OffBar + A_NUM * 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  int* n_pieces = reinterpret_cast<int*>(misc + 8);
  Piece* pcs = reinterpret_cast<Piece*>(misc + 16);
  auto bar = [&](int i) { return base + kA_OffBar + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < A_NUM; ++i)
      mbar_init(bar(i), (i == A_S_EMPTY || i == A_S_EMPTY + 1) ? 128u * kWg : 1u);   // every softmax thread
    *abort_flag = 0;
    *n_pieces = build_pieces(p, pcs);
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
  // the cache, the workspace and the counters may still be in use by the previous kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");
  int npc = *n_pieces;
  if (npc < 0) {
    if (threadIdx.x == 0) atomicOr(p.err, kErrBounds);
    npc = 0;
  }
  if (threadIdx.x == 0)   // kernel B counts the pieces of each unit from zero
    for (int i = 0; i < npc; ++i)
      if (pcs[i].k == 0) p.count[pcs[i].u] = 0;

  if (warp == 0) {
    // =========================================================== TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_kc);
      bool ok = true;
      int tc = 0, q_issued = 0;
      for (int pi = 0; ok && pi < npc; ++pi) {
        const Piece x = pcs[pi];
        const UnitGeo g = unit_geo(p, x.u);
        if (pi > 0) ok = mbar_wait(bar(A_Q_EMPTY), (uint32_t)(pi - 1) & 1u, abort_flag, p.err,
                                   kWaitLimitNs, kErrTimeout);
        if (!ok) break;
        const int zq = g.b * p.Hq + g.h * p.G + g.gl_a;
        mbar_arrive_expect_tx(bar(A_Q), 2 * kTile);
        for (int hw = 0; hw < 2; ++hw)
          for (int at = 0; at < 2; ++at)
            tma_load_3d(base + kA_OffQ + at * 2 * kAtom + hw * kAtom, &tm_q, bar(A_Q), at * 64,
                        (int)g.i0, zq + hw);
        q_issued = pi + 1;
        for (int pr = x.a; ok && pr < x.c; ++pr) {
          const int s = tc & 1;
          ok = mbar_wait(bar(A_K_EMPTY + s), ((uint32_t)(tc >> 1) & 1u) ^ 1u, abort_flag, p.err,
                         kWaitLimitNs, kErrTimeout);
          if (!ok) break;
          const uint32_t dst = base + kA_OffK + (uint32_t)s * kA_Slot;
          mbar_arrive_expect_tx(bar(A_K_FULL + s), kA_Slot);
          for (int half = 0; half < 2; ++half) {
            const int t = 2 * pr + half;
            const CUtensorMap* m = t < g.nct ? &tm_kc : &tm_k;
            // past the unit's last tile: a box beyond the chunk's rows reads zeros
            const int y = t < g.nct ? t * BN : (t < g.n_all ? (t - g.nct) * BN : (int)p.S);
            for (int at = 0; at < 2; ++at)
              tma_load_3d(dst + at * 2 * kAtom + half * kAtom, m, bar(A_K_FULL + s), at * 64, y, g.bh);
          }
          ++tc;
        }
      }
      // drain, also after an abort: every load issued has landed
      if (q_issued > 0) mbar_drain(bar(A_Q), (uint32_t)(q_issued - 1) & 1u, p.err, kWaitLimitNs, kErrTimeout);
      for (int t = tc - 2 < 0 ? 0 : tc - 2; t < tc; ++t)
        mbar_drain(bar(A_K_FULL + (t & 1)), (uint32_t)(t >> 1) & 1u, p.err, kWaitLimitNs, kErrTimeout);
    }
  } else if (warp == 1) {
    // =========================================================== MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, 256, 0, 0);   // both operands K-major
      const uint32_t q_addr = base + kA_OffQ;
      bool ok = true;
      int tc = 0;
      for (int pi = 0; ok && pi < npc; ++pi) {
        const Piece x = pcs[pi];
        ok = mbar_wait(bar(A_Q), (uint32_t)pi & 1u, abort_flag, p.err, kWaitLimitNs, kErrTimeout);
        for (int pr = x.a; ok && pr < x.c; ++pr) {
          const int s = tc & 1;
          ok = mbar_wait(bar(A_K_FULL + s), (uint32_t)(tc >> 1) & 1u, abort_flag, p.err, kWaitLimitNs,
                         kErrTimeout);
          const uint32_t k_addr = base + kA_OffK + (uint32_t)s * kA_Slot;
          for (int w = 0; ok && w < 2; ++w) {
            ok = mbar_wait(bar(A_S_EMPTY + w), ((uint32_t)tc & 1u) ^ 1u, abort_flag, p.err,
                           kWaitLimitNs, kErrTimeout);
            if (!ok) break;
            tc_fence_after();
            const uint32_t a0 = desc_lo(q_addr + (uint32_t)w * kAtom, 16), b0 = desc_lo(k_addr, 16);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              umma_bf16(tmem + (uint32_t)w * 256u, a0 + (kmajor_off(kk, 256) >> 4), kDescHi,
                        b0 + (kmajor_off(kk, 256) >> 4), kDescHi, idesc, kk > 0 ? 1u : 0u);
            umma_commit(bar(A_S_FULL + w));
          }
          if (ok) umma_commit(bar(A_K_EMPTY + s));
          ++tc;
        }
        if (ok) umma_commit(bar(A_Q_EMPTY));   // Q is free once this piece's MMAs are done
      }
      // every MMA issued has completed before TMEM is released, also after an abort
      umma_commit(bar(A_DRAIN));
      mbar_drain(bar(A_DRAIN), 0, p.err, kWaitLimitNs, kErrTimeout);
    }
  } else {
    // =========================================================== softmax: row (max, sum)
    // Four warpgroups read each head's S tile, warpgroup g taking keys
    // [64 g, 64 g + 64) of every 256-key tile (four warps per SM sub-partition
    // hide each other's latencies; a tile is released as soon as it is loaded
    // into registers); thread = query row r of both heads.  At the end of a
    // piece warpgroup w < 2 merges the four (max, sum) of head w's rows, in
    // warpgroup order, and writes them.
    const int wg = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                 // TMEM lane = query row
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)wg * 64u;
    const float c = p.scale_log2;
    const int64_t S = p.S, nv = p.n_valid;
    float2* mrg = reinterpret_cast<float2*>(sbase + kA_OffMrg);
    bool ok = true;
    int tc = 0;
    for (int pi = 0; pi < npc; ++pi) {
      const Piece x = pcs[pi];
      const UnitGeo g = unit_geo(p, x.u);
      const int64_t row_i = g.i0 + r;
      const int64_t row_lim = (row_i + 1 < S) ? row_i + 1 : S;   // chunk keys < row_lim are seen
      auto nvis_of = [&](int t, int half64) -> int {
        if (t >= g.n_all) return 0;
        const bool cache = t < g.nct;
        const int64_t key0 = (cache ? (int64_t)t * BN : (int64_t)(t - g.nct) * BN) + half64 * 64;
        const int64_t lim = cache ? nv : row_lim;
        return (int)(lim - key0 > 64 ? 64 : (lim - key0 < 0 ? 0 : lim - key0));
      };
      float mh[2] = {-INFINITY, -INFINITY}, lh[2] = {0.f, 0.f};
      for (int pr = x.a; ok && pr < x.c; ++pr) {
#pragma unroll
        for (int hw = 0; hw < 2; ++hw) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar(A_S_FULL + hw), (uint32_t)tc & 1u, abort_flag, p.err,
                                                 kWaitLimitNs, kErrTimeout));
          if (!ok) break;
          tc_fence_after();
          uint32_t v[2][32];
          tmem_ld32(lane_base + (uint32_t)hw * 256u, v[0]);
          tmem_ld32(lane_base + (uint32_t)hw * 256u + 32u, v[1]);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(bar(A_S_EMPTY + hw));
          row_chunk(v, nvis_of(2 * pr + (wg >> 1), wg & 1), c, mh[hw], lh[hw]);
        }
        __syncwarp();
        ++tc;
      }
      // Every warp passes both barriers whatever its `ok`, and the second one
      // makes the decision to stop the same for all of them.
      mrg[(wg * 2 + 0) * BM + r] = make_float2(mh[0], lh[0]);
      mrg[(wg * 2 + 1) * BM + r] = make_float2(mh[1], lh[1]);
      named_bar_sync(1, kSoft);
      float m = -INFINITY, l = 0.f;
      if (wg < 2) {
        float2 o[kWg];
#pragma unroll
        for (int q = 0; q < kWg; ++q) {
          o[q] = mrg[(q * 2 + wg) * BM + r];
          m = fmaxf(m, o[q].x);
        }
        // an empty part has sum 0 (or NaN when its keys were all masked)
#pragma unroll
        for (int q = 0; q < kWg; ++q)
          if (o[q].y > 0.f) l += o[q].y * ex2(o[q].x - m);
      }
      ok = named_bar_and(1, kSoft, ok);   // all read: the next piece may overwrite the area
      if (!ok) break;
      if (wg < 2) p.ws_ml[((int64_t)x.u * p.maxp + x.k) * (2 * BM) + wg * BM + r] = make_float2(m, l);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ kernel B
__global__ void __launch_bounds__(kThreads, 1)
attn_stream_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kc,
                   const __grid_constant__ CUtensorMap tm_vc, const SParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  float* nlse = reinterpret_cast<float*>(sbase + kB_OffLse);
  uint8_t* misc = sbase + kB_OffBar + B_NUM * 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  int* n_pieces = reinterpret_cast<int*>(misc + 8);
  volatile int* last_flag = reinterpret_cast<volatile int*>(misc + 12);
  Piece* pcs = reinterpret_cast<Piece*>(misc + 16);
  auto bar = [&](int i) { return base + kB_OffBar + 8u * (uint32_t)i; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < B_NUM; ++i) {
      uint32_t cnt = 1;
      if (i == B_P_FULL || i == B_O_EMPTY) cnt = kSoft;                  // every softmax thread
      if (i == B_ST_EMPTY || i == B_ST_EMPTY + 1) cnt = kSoft / 2;        // one head's warpgroups
      mbar_init(bar(i), cnt);
    }
    *abort_flag = 0;
    *n_pieces = build_pieces(p, pcs);
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
  // kernel A's workspace and counters are complete once the previous grid is
  asm volatile("griddepcontrol.wait;" ::: "memory");
  int npc = *n_pieces;
  if (npc < 0) {
    if (threadIdx.x == 0) atomicOr(p.err, kErrBounds);
    npc = 0;
  }
  // a piece's tiles [t_lo, t_hi) of its unit
  auto piece_tiles = [&](const Piece& x, const UnitGeo& g, int& t_lo, int& n) {
    t_lo = 2 * x.a;
    const int t_hi = 2 * x.c < g.n_all ? 2 * x.c : g.n_all;
    n = t_hi - t_lo;
  };

  if (warp == 0) {
    // =========================================================== TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_kc);
      prefetch_tmap(&tm_vc);
      bool ok = true;
      int gp = 0, q_issued = 0;                      // ring positions issued, over all pieces
      for (int pi = 0; ok && pi < npc; ++pi) {
        const Piece x = pcs[pi];
        const UnitGeo g = unit_geo(p, x.u);
        int t_lo, n;
        piece_tiles(x, g, t_lo, n);
        if (pi > 0) ok = mbar_wait(bar(B_Q_EMPTY), (uint32_t)(pi - 1) & 1u, abort_flag, p.err,
                                   kWaitLimitNs, kErrTimeout);
        if (!ok) break;
        const int zq = g.b * p.Hq + g.h * p.G + g.gl_a;
        mbar_arrive_expect_tx(bar(B_Q), 2 * kTile);
        for (int hw = 0; hw < 2; ++hw)
          for (int at = 0; at < 2; ++at)
            tma_load_3d(base + kB_OffQ + at * 2 * kAtom + hw * kAtom, &tm_q, bar(B_Q), at * 64,
                        (int)g.i0, zq + hw);
        q_issued = pi + 1;
        for (int pos = 0; ok && pos < 2 * n; ++pos) {
          const int slot = gp % NS2;
          ok = mbar_wait(bar(B_R_EMPTY + slot), ((uint32_t)(gp / NS2) & 1u) ^ 1u, abort_flag, p.err,
                         kWaitLimitNs, kErrTimeout);
          if (!ok) break;
          bool is_v;
          int t;
          if (pos == 0) { is_v = false; t = 0; }
          else if (pos == 2 * n - 1) { is_v = true; t = n - 1; }
          else if (pos & 1) { is_v = false; t = (pos + 1) >> 1; }
          else { is_v = true; t = (pos >> 1) - 1; }
          const int tg = t_lo + t;
          const CUtensorMap* m = tg < g.nct ? (is_v ? &tm_vc : &tm_kc) : (is_v ? &tm_v : &tm_k);
          const int y = tg < g.nct ? tg * BN : (tg - g.nct) * BN;
          const uint32_t dst = base + kB_OffR + (uint32_t)slot * kTile;
          mbar_arrive_expect_tx(bar(B_R_FULL + slot), kTile);
          tma_load_3d(dst, m, bar(B_R_FULL + slot), 0, y, g.bh);
          tma_load_3d(dst + kAtom, m, bar(B_R_FULL + slot), 64, y, g.bh);
          ++gp;
        }
      }
      // drain, also after an abort: every load issued has landed
      if (q_issued > 0) mbar_drain(bar(B_Q), (uint32_t)(q_issued - 1) & 1u, p.err, kWaitLimitNs, kErrTimeout);
      for (int pos = gp - NS2 < 0 ? 0 : gp - NS2; pos < gp; ++pos)
        mbar_drain(bar(B_R_FULL + pos % NS2), (uint32_t)(pos / NS2) & 1u, p.err, kWaitLimitNs,
                   kErrTimeout);
    }
  } else if (warp == 1) {
    // =========================================================== MMA issuer
    if (lane == 0) {
      const uint32_t idesc_st = idesc_bf16(128, 128, 0, 0);   // S^T of one head: K-major operands
      const uint32_t idesc_mn = idesc_bf16(128, 256, 1, 1);   // O^T: both operands MN-major
      const uint32_t q_addr = base + kB_OffQ;
      const uint32_t p_addr = base + kB_OffP;
      bool ok = true;
      int gp_base = 0, st = 0, ot = 0;                // over all pieces
      for (int pi = 0; ok && pi < npc; ++pi) {
        const Piece x = pcs[pi];
        const UnitGeo g = unit_geo(p, x.u);
        int t_lo, n;
        piece_tiles(x, g, t_lo, n);
        ok = mbar_wait(bar(B_Q), (uint32_t)pi & 1u, abort_flag, p.err, kWaitLimitNs, kErrTimeout);
        auto issue_st = [&](int j) -> bool {
          const int pos = gp_base + k_pos(j), slot = pos % NS2;
          if (!mbar_wait(bar(B_R_FULL + slot), (uint32_t)(pos / NS2) & 1u, abort_flag, p.err, kWaitLimitNs,
                         kErrTimeout))
            return false;
          const uint32_t k_addr = base + kB_OffR + (uint32_t)slot * kTile;
          for (int hh = 0; hh < 2; ++hh) {
            // head hh's S^T buffer must have been read by its two warpgroups
            if (st > 0 && !mbar_wait(bar(B_ST_EMPTY + hh), (uint32_t)(st - 1) & 1u, abort_flag, p.err,
                                     kWaitLimitNs, kErrTimeout))
              return false;
            tc_fence_after();
            const uint32_t a0 = desc_lo(k_addr, 16), b0 = desc_lo(q_addr + (uint32_t)hh * 16384u, 16);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              umma_bf16(tmem + (uint32_t)hh * 128u, a0 + (kmajor_off(kk, 128) >> 4), kDescHi,
                        b0 + (kmajor_off(kk, 256) >> 4), kDescHi, idesc_st, kk > 0 ? 1u : 0u);
            umma_commit(bar(B_ST_FULL + hh));
          }
          umma_commit(bar(B_R_EMPTY + slot));
          ++st;
          return true;
        };
        auto issue_ot = [&](int j) -> bool {
          bool w_ok = mbar_wait(bar(B_P_FULL), (uint32_t)ot & 1u, abort_flag, p.err, kWaitLimitNs,
                                kErrTimeout);
          // the first O^T MMA of a piece overwrites TMEM columns 256-511: the
          // softmax must have read the previous piece's O^T
          if (w_ok && j == 0 && pi > 0)
            w_ok = mbar_wait(bar(B_O_EMPTY), (uint32_t)(pi - 1) & 1u, abort_flag, p.err, kWaitLimitNs,
                             kErrTimeout);
          const int pos = gp_base + v_pos(n, j), slot = pos % NS2;
          if (w_ok)
            w_ok = mbar_wait(bar(B_R_FULL + slot), (uint32_t)(pos / NS2) & 1u, abort_flag, p.err,
                             kWaitLimitNs, kErrTimeout);
          if (!w_ok) return false;
          tc_fence_after();
          const uint32_t a0 = desc_lo(base + kB_OffR + (uint32_t)slot * kTile, kAtom), b0 = desc_lo(p_addr, kAtom);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            umma_bf16(tmem + 256u, a0 + (uint32_t)kk * 128u, kDescHi, b0 + (uint32_t)kk * 128u, kDescHi, idesc_mn,
                      (j > 0 || kk > 0) ? 1u : 0u);
          umma_commit(bar(B_P_EMPTY));
          umma_commit(bar(B_R_EMPTY + slot));
          ++ot;
          return true;
        };
        for (int j = 0; ok && j < n; ++j) {
          ok = issue_st(j);
          if (ok && j == n - 1) umma_commit(bar(B_Q_EMPTY));   // Q is free once the last S^T is done
          if (ok && j > 0) ok = issue_ot(j - 1);
        }
        if (ok) ok = issue_ot(n - 1);
        if (ok) umma_commit(bar(B_O_FULL));
        gp_base += 2 * n;
      }
      // every MMA issued has completed before TMEM is released, also after an abort
      umma_commit(bar(B_DRAIN));
      mbar_drain(bar(B_DRAIN), 0, p.err, kWaitLimitNs, kErrTimeout);
    }
  } else {
    // =========================================================== softmax / epilogue
    // Four warpgroups: warpgroup wg takes the 64 query columns [64 wg, 64 wg + 64)
    // of S^T, i.e. queries [64 hq, 64 hq + 64) of head w (w = wg / 2, hq = wg % 2),
    // and adds its column sums of them to the accumulator row.
    const int wg = (warp - 2) >> 2;
    const int w = wg >> 1, hq = wg & 1;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                 // TMEM lane: key in S^T, d in O^T
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t st_tmem = lane_base + (uint32_t)wg * 64u;
    const uint32_t o_tmem = lane_base + 256u + (uint32_t)wg * 64u;
    const uint32_t p_row = base + kB_OffP + (uint32_t)wg * kAtom + (uint32_t)(r >> 3) * 1024u +
                           (uint32_t)(r & 7) * 128u;
    const float* nl_w = nlse + wg * 64;
    const int64_t S = p.S, M = p.M, nv = p.n_valid;
    const float c = p.scale_log2;
    const int t = threadIdx.x - 64;                    // 0 .. kSoft-1 over all warpgroups
    bool ok = true;
    int st = 0;
    if (p.inject_timeout && wg == 0) {
      // test hook: a bounded wait on a barrier nothing completes runs out (1 ms);
      // every role then leaves through its abort path and the step reports it
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_NEVER), 0, abort_flag, p.err, 1000000ull, kErrTimeout));
    }
    // every warp passes every named barrier below whatever its `ok`, so a warp
    // that aborted cannot leave the others waiting; only the work is skipped
    for (int pi = 0; pi < npc; ++pi) {
      const Piece x = pcs[pi];
      const UnitGeo g = unit_geo(p, x.u);
      int t_lo, n;
      piece_tiles(x, g, t_lo, n);
      const bool head_ok = w == 0 || g.has_b;
      // the unit's log-sum-exp of row r of head wg (wg < 2): its pieces' (max, sum) in piece order
      named_bar_sync(1, kSoft);                        // the previous piece is done with nlse
      if (ok && wg < 2) {
        const float2* ml = p.ws_ml + (int64_t)x.u * p.maxp * (2 * BM) + wg * BM + r;
        float mx = -INFINITY;
        for (int k = 0; k < x.np; ++k) {
          const float2 v = ml[(int64_t)k * (2 * BM)];
          if (v.y > 0.f) mx = fmaxf(mx, v.x);
        }
        float lsum = 0.f;
        for (int k = 0; k < x.np; ++k) {
          const float2 v = ml[(int64_t)k * (2 * BM)];
          if (v.y > 0.f) lsum += v.y * ex2(v.x - mx);
        }
        const int64_t row_i = g.i0 + r;
        const bool row_head_ok = wg == 0 || g.has_b;
        nlse[wg * BM + r] = (row_head_ok && row_i < S && lsum > 0.f) ? -(mx + lg2(lsum)) : -INFINITY;
      }
      named_bar_sync(1, kSoft);
      unsigned long long* acc = p.colacc + (int64_t)g.bh * p.acc_stride;
      for (int j = 0; ok && j < n; ++j) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(B_ST_FULL + w), (uint32_t)st & 1u, abort_flag, p.err,
                                               kWaitLimitNs, kErrTimeout));
        if (!ok) break;
        tc_fence_after();
        const int jg = t_lo + j;
        const bool cache = jg < g.nct;
        const int64_t key = cache ? (int64_t)jg * BN + r : (int64_t)(jg - g.nct) * BN + r;
        const bool key_ok = cache ? key < nv : key < S;
        // chunk key `key` is seen by query columns q with i0 + q >= key
        const int qmin = (cache ? 0 : (int)(key - g.i0 > 0 ? key - g.i0 : 0)) - 64 * hq;
        const bool full = __all_sync(0xffffffffu, key_ok && qmin <= 0);
        uint64_t cs4[4] = {0ull, 0ull, 0ull, 0ull};
        // the key's 64 probabilities in registers before waiting for the P^T
        // buffer, so the previous tile's O^T MMA overlaps the exponentials
        uint32_t pk[32];
#pragma unroll
        for (int qc = 0; qc < 2; ++qc) {
          uint32_t v[32];
          tmem_ld32(st_tmem + qc * 32, v);
          tmem_wait_ld();
          if (qc == 1) {
            tc_fence_before();
            mbar_arrive(bar(B_ST_EMPTY + w));
          }
          if (full) key_part<true, 32>(v, nl_w + qc * 32, c, key_ok, qmin - qc * 32, cs4, pk + qc * 16);
          else key_part<false, 32>(v, nl_w + qc * 32, c, key_ok, qmin - qc * 32, cs4, pk + qc * 16);
        }
        ok = __all_sync(0xffffffffu, mbar_wait(bar(B_P_EMPTY), ((uint32_t)st & 1u) ^ 1u, abort_flag,
                                               p.err, kWaitLimitNs, kErrTimeout));
        if (!ok) break;
        store_p_half(p_row, r, pk);
        fence_async_smem();
        mbar_arrive(bar(B_P_FULL));
        // without a head B every p of warpgroups 2 and 3 is 0
        if (key_ok && head_ok) colsum_add(acc + (cache ? key : M + key), cs_total(cs4), p.fx_scale);
        ++st;
      }
      // ----- the piece's O^T (lane = d, columns = the warpgroup's 64 queries of head w)
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_O_FULL), (uint32_t)pi & 1u, abort_flag, p.err,
                                                     kWaitLimitNs, kErrTimeout));
      if (ok) tc_fence_after();
      const int gq = g.h * p.G + g.gl_a + w;           // query head of warpgroup wg
      float* wsp = p.ws_o + (((int64_t)x.u * p.maxp + x.k) * (2 * BM) + wg * 64) * D;
#pragma unroll 1
      for (int ch = 0; ok && ch < 2; ++ch) {
        uint32_t o[32];
        tmem_ld32(o_tmem + ch * 32, o);
        tmem_wait_ld();
        if (x.np == 1) {
          if (p.out != nullptr && head_ok) {
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + ((int64_t)g.b * p.Hq + gq) * S * D + r;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              const int64_t qi = g.i0 + 64 * hq + ch * 32 + k;
              if (qi < S) dst[qi * D] = __float2bfloat16_rn(__uint_as_float(o[k]));
            }
          }
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) wsp[(ch * 32 + k) * D + r] = __uint_as_float(o[k]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(B_O_EMPTY));                     // TMEM O^T may be overwritten
      if (x.np > 1 && p.out != nullptr) {
        // the last piece of the unit to get here adds all partials in piece order
        __threadfence();
        named_bar_sync(3, kSoft);
        if (t == 0) *last_flag = atomicAdd(p.count + x.u, 1) == x.np - 1;
        named_bar_sync(3, kSoft);
        if (*last_flag) {
          __threadfence();
          const float* ws0 = p.ws_o + (int64_t)x.u * p.maxp * (2 * BM) * D;
          // items (query q, 8 values of d from d0): four at a time, so that each
          // thread has 8 loads per piece in flight
          constexpr int kItems = 2 * BM * (D / 8);
          static_assert(kItems % (4 * kSoft) == 0, "whole rounds of items");
          for (int it0 = t; it0 < kItems; it0 += 4 * kSoft) {
            float4 lo[4], hi[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) lo[i] = hi[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int k = 0; k < x.np; ++k) {
              float4 a[4], b2[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int it = it0 + i * kSoft;
                const float4* src = reinterpret_cast<const float4*>(
                    ws0 + ((int64_t)k * (2 * BM) + it / (D / 8)) * D + (it % (D / 8)) * 8);
                a[i] = __ldcg(src);
                b2[i] = __ldcg(src + 1);
              }
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                lo[i].x += a[i].x; lo[i].y += a[i].y; lo[i].z += a[i].z; lo[i].w += a[i].w;
                hi[i].x += b2[i].x; hi[i].y += b2[i].y; hi[i].z += b2[i].z; hi[i].w += b2[i].w;
              }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int it = it0 + i * kSoft;
              const int q = it / (D / 8), d0 = (it % (D / 8)) * 8;
              const int wq = q / BM;
              const int64_t qi = g.i0 + (q % BM);
              if ((wq == 0 || g.has_b) && qi < S) {
                uint4 v;
                v.x = pack_bf16(lo[i].x, lo[i].y);
                v.y = pack_bf16(lo[i].z, lo[i].w);
                v.z = pack_bf16(hi[i].x, hi[i].y);
                v.w = pack_bf16(hi[i].z, hi[i].w);
                const int gh = g.h * p.G + g.gl_a + wq;
                *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                          (((int64_t)g.b * p.Hq + gh) * S + qi) * D + d0) = v;
              }
            }
          }
          if (t == 0) p.count[x.u] = 0;
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

}  // namespace

// (b, KV head) caches per round: all of them when their K and V rows (those
// the step reads) fit in three quarters of L2; otherwise as many as fit in
// half of it, at least one, in rounds of equal size.  (Measured on B200: one
// round at 16k slots, where the eight heads' 71 MB fit; three rounds at 32k
// slots, 142 MB.)
int heads_per_round(const AttnArgs& a) {
  const int BH = a.B * a.Hkv;
  int l2 = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess) {
    cudaGetLastError();
    return BH;
  }
  const double kv = (double)(a.n_valid + a.S) * D * 2.0 * 2.0;   // bf16 K and V of one cache
  if (BH * kv <= 0.75 * l2) return BH;
  int h = (int)(0.5 * l2 / kv);
  if (h < 1) h = 1;
  if (h >= BH) return BH;
  const int rounds = (BH + h - 1) / h;
  return (BH + rounds - 1) / rounds;
}

bool attn_stream_plan(const AttnArgs& a, int n_sm, StreamPlan* pl) {
  if (!attn_umma_supported(kBF16, a.d) || n_sm < 1 || a.S < 1) return false;
  const int G = a.Hq / a.Hkv, n_pg = (G + 1) / 2;
  const int n_rt = (int)((a.S + BM - 1) / BM);
  const int BH = a.B * a.Hkv, per_head = n_pg * n_rt;
  const int64_t units = (int64_t)BH * per_head;
  if (units < 1 || units > (1 << 24)) return false;
  const int nct = (int)((a.n_valid + BN - 1) / BN);
  std::vector<int> q((size_t)units);
  int64_t P = 0;
  for (int64_t u = 0; u < units; ++u) {
    const int rt = (int)(u % n_rt);
    const int64_t i0 = (int64_t)rt * BM, chunk_hi = i0 + BM < a.S ? i0 + BM : a.S;
    const int n_all = nct + (int)((chunk_hi + BN - 1) / BN);
    q[(size_t)u] = (n_all + 1) >> 1;
    P += q[(size_t)u];
  }
  const int hpr = heads_per_round(a);
  // every round is cut into n_cta runs; with fewer pairs than SMs in a round,
  // n_cta is that round's pair count at most
  int n_cta = n_sm;
  for (int h0 = 0; h0 < BH; h0 += hpr) {
    int64_t Pr = 0;
    for (int u = h0 * per_head; u < (h0 + hpr < BH ? h0 + hpr : BH) * per_head; ++u) Pr += q[(size_t)u];
    if (Pr < n_cta) n_cta = (int)Pr;
  }
  std::vector<int> per_cta((size_t)n_cta, 0);
  int maxp = 1;
  for (int h0 = 0; h0 < BH; h0 += hpr) {
    const int u_lo = h0 * per_head, u_hi = (h0 + hpr < BH ? h0 + hpr : BH) * per_head;
    int64_t Pr = 0;
    for (int u = u_lo; u < u_hi; ++u) Pr += q[(size_t)u];
    int64_t g0 = 0;
    for (int u = u_lo; u < u_hi; ++u) {
      const int first = cta_of(g0, Pr, n_cta), last = cta_of(g0 + q[(size_t)u] - 1, Pr, n_cta);
      if (last - first + 1 > maxp) maxp = last - first + 1;
      for (int i = first; i <= last; ++i)
        if (++per_cta[(size_t)i] > kMaxPieces) return false;
      g0 += q[(size_t)u];
    }
  }
  pl->n_cta = n_cta;
  pl->maxp = maxp;
  pl->units = (int)units;
  pl->total_pairs = P;
  pl->heads_per_round = hpr;
  pl->ml_bytes = (size_t)units * maxp * 2 * BM * sizeof(float2);
  pl->o_bytes = maxp > 1 ? (size_t)units * maxp * 2 * BM * D * sizeof(float) : 0;
  pl->count_bytes = (size_t)units * sizeof(int);
  return true;
}

cudaError_t launch_attn_stream(const AttnArgs& a, const StreamPlan& pl, void* ws_ml, void* ws_o,
                               int* count, bool pdl, cudaStream_t st) {
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
  SParams p;
  p.colacc = a.colacc;
  p.err = a.err;
  p.out = a.out;
  p.ws_ml = static_cast<float2*>(ws_ml);
  p.ws_o = static_cast<float*>(ws_o);
  p.count = count;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.n_pg = (p.G + 1) / 2;
  p.n_rt = (int)((a.S + BM - 1) / BM);
  p.maxp = pl.maxp;
  p.inject_timeout = a.inject_timeout;
  p.S = a.S;
  p.M = a.M;
  p.n_valid = a.n_valid;
  p.acc_stride = a.acc_stride;
  p.fx_scale = fx_scale_of(a.fx_shift);
  p.heads_per_round = pl.heads_per_round;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  if ((e = cudaFuncSetAttribute(lse_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kA_SmemBytes)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(attn_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kB_SmemBytes)) != cudaSuccess)
    return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)pl.n_cta);
  cfg.blockDim = dim3(kThreads);
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  cfg.dynamicSmemBytes = kA_SmemBytes;
  cfg.blockDim = dim3(kThreads);
  if ((e = cudaLaunchKernelEx(&cfg, lse_stream_kernel, mq, mk, mkc, p)) != cudaSuccess) return e;
  cfg.blockDim = dim3(kThreads);
  at[0].val.programmaticStreamSerializationAllowed = 1;   // kernel B follows kernel A
  cfg.dynamicSmemBytes = kB_SmemBytes;
  return cudaLaunchKernelEx(&cfg, attn_stream_kernel, mq, mk, mv, mkc, mvc, p);
}

}  // namespace h2o
