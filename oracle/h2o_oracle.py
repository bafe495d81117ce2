"""Float64 CPU oracle for the H2O chunk step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py`` may import this module.  The product
path (``h2o_kv_cache_b200``) never imports, calls or links it, and this module
imports nothing from the product path.

Source: "Learning how to Forget: Fine-tuning for Long-Context Sparse Attention"
(Seeger, Zhang, Patil, Benidis, Schelter).
  * Abstract: an implementation of H2O sparse attention with a dedicated scaled
    dot product attention (SDPA) kernel.
  * §1 Introduction, ¶1: key-value information lives in a fixed-size KV cache
    whose slots are evicted once it is full.
  * §1 Introduction, ¶3: usable with grouped query attention.
  * §1 Introduction, ¶4: H2O is the heavy-hitter oracle.
  * FAQ, answer 3: the SDPA kernel also returns the summed attention weights.
  * Figure 1(a): the computation is a lattice of chunks -- a prefill chunk of
    full length N_C, then chunks of length S << N_C.

The pages give no formulas for the policy.  The steps below are the plainest
reading of the method as the pages name it; every reading of an open point is
written next to the code that takes it:

  state per (batch b, KV head h): K, V [M, d]; score [M]; pos [M] (-1 = empty)
  step with a chunk of S tokens at stream offset t0:
    1. attend   -- every query row (g, i) of the KV head's group sees all valid
                   slots plus chunk keys j <= i; p = softmax(q.k / sqrt(d));
                   out = p . V
    2. summed weights -- c_j = sum over the group's query heads and the chunk's
                   queries of p_ij, for every slot and every chunk key
    3. accumulate -- score[valid slot] += c_slot
    4. evict    -- need = max(0, S - #empty); among valid slots with
                   pos < t0 - R pick the `need` smallest by (score, pos)
    5. scatter  -- freed = ascending(evicted + first S-need empty slots);
                   chunk token i -> freed[i]: K/V row, pos = t0 + i,
                   score = c_{chunk key i}
  prefill = the same step on an empty cache (no eviction).

All pins of this module (tests/test_oracle.py) reach it from outside: a
hand-worked 8-token example in exact fractions, the invariant that each chunk
adds S*G of mass per KV head, exact causal attention from a library routine when
the cache never fills, an independent position-indexed brute force, and the
selection against numpy's lexsort.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "attend_group",
    "select_evictions",
    "select_oldest",
    "H2OHeadOracle",
    "H2OOracle",
    "OracleShapeError",
]


class OracleShapeError(ValueError):
    """The step cannot be taken: too few evictable slots, or P > M."""


def attend_group(q_g, k_slots, v_slots, slot_valid, k_new, v_new, scale, row_block=512):
    """SDPA over the valid cache slots plus the chunk's own keys, with summed weights.

    Follows the pages' "SDPA kernel ... plus code to return summed attention
    weights" (FAQ, answer 3) over the fixed-size cache of §1 ¶1; GQA as in §1 ¶3.

    q_g       [G, S, d]  the G query heads that share this KV head
    k_slots   [M, d], v_slots [M, d]  cache contents (rows of invalid slots ignored)
    slot_valid [M] bool
    k_new, v_new [S, d]  the chunk's own keys / values (causal: key j seen by rows i >= j)
    Returns   out [G, S, d] float64, c_slots [M] (0 for invalid slots), c_new [S]

    Softmax is exact in float64: each row's logits are shifted by the row max,
    exponentiated and divided by their sum.  Rows are processed in blocks only to
    bound memory; nothing is reordered across a row.
    """
    q_g = np.asarray(q_g, dtype=np.float64)
    G, S, d = q_g.shape
    M = k_slots.shape[0]
    valid_idx = np.nonzero(np.asarray(slot_valid))[0]
    n_c = valid_idx.size
    keys = np.concatenate([np.asarray(k_slots, np.float64)[valid_idx],
                           np.asarray(k_new, np.float64)], axis=0)      # [n_c + S, d]
    vals = np.concatenate([np.asarray(v_slots, np.float64)[valid_idx],
                           np.asarray(v_new, np.float64)], axis=0)
    out = np.zeros((G, S, d), dtype=np.float64)
    colsum = np.zeros(n_c + S, dtype=np.float64)
    # causal visibility of chunk key j for row i: j <= i
    jj = np.arange(S)
    for g in range(G):
        for r0 in range(0, S, row_block):
            r1 = min(S, r0 + row_block)
            logits = (q_g[g, r0:r1] @ keys.T) * scale                     # [rows, n_c + S]
            ii = np.arange(r0, r1)[:, None]
            hidden = jj[None, :] > ii                                     # chunk keys after the row
            logits[:, n_c:][hidden] = -np.inf
            m = logits.max(axis=1, keepdims=True)
            e = np.exp(logits - m)
            p = e / e.sum(axis=1, keepdims=True)
            out[g, r0:r1] = p @ vals
            colsum += p.sum(axis=0)
    c_slots = np.zeros(M, dtype=np.float64)
    c_slots[valid_idx] = colsum[:n_c]
    return out, c_slots, colsum[n_c:]


def select_evictions(score, pos, t0, R, need):
    """Slots to evict: the `need` smallest eligible slots by (score, pos), ascending by slot.

    Eligible: a valid slot (pos >= 0) whose token is older than the protected
    recent window, i.e. pos < t0 - R.  Reading (pages silent): the window is the
    R most recent tokens *before* the chunk, and ties in score go to the older
    token (lower pos evicted first).
    Written as a plain Python sort on (score, pos) tuples.
    """
    score = np.asarray(score, dtype=np.float64)
    pos = np.asarray(pos)
    eligible = [s for s in range(score.shape[0]) if pos[s] >= 0 and pos[s] < t0 - R]
    if need > len(eligible):
        raise OracleShapeError(f"need {need} evictions but only {len(eligible)} eligible slots")
    ranked = sorted(eligible, key=lambda s: (float(score[s]), int(pos[s])))
    return sorted(ranked[:need])


def select_oldest(pos, t0, R, need):
    """Slots to evict under the recency-only policy: the `need` eligible slots
    holding the oldest tokens (smallest pos), ascending by slot.

    The page names an `lr` policy beside `h2o` (Tables 1 and 6) without
    defining it; the reading taken is the plainest one for its name: keep the
    most recent tokens.  Eligibility is the same as for H2O (valid, and older
    than the protected recent window).  Written as a plain Python sort on pos.
    """
    pos = np.asarray(pos)
    eligible = [s for s in range(pos.shape[0]) if pos[s] >= 0 and pos[s] < t0 - R]
    if need > len(eligible):
        raise OracleShapeError(f"need {need} evictions but only {len(eligible)} eligible slots")
    ranked = sorted(eligible, key=lambda s: int(pos[s]))
    return sorted(ranked[:need])


class H2OHeadOracle:
    """State and step of one (batch, KV head) cache; eviction is per KV head.
    policy "h2o" (heavy hitters, the default) or "lr" (recency only)."""

    def __init__(self, M, R, G, d, policy="h2o"):
        if policy not in ("h2o", "lr"):
            raise ValueError(f"unknown policy {policy!r}")
        self.policy = policy
        self.M, self.R, self.G, self.d = int(M), int(R), int(G), int(d)
        self.K = np.zeros((self.M, self.d), dtype=np.float64)
        self.V = np.zeros((self.M, self.d), dtype=np.float64)
        self.score = np.zeros(self.M, dtype=np.float64)
        self.pos = np.full(self.M, -1, dtype=np.int64)
        self.t0 = 0
        # diagnostics of the last step, read by the parity harness
        self.last_freed = None
        self.last_pre_scores = None    # scores after accumulate, before eviction
        self.last_eligible = None
        self.last_need = 0
        self.last_c_slots = None
        self.last_c_new = None

    def load_state(self, K, V, score, pos, t0):
        """Overwrite the state (used to re-synchronise at tie-consistent boundaries)."""
        self.K = np.array(K, dtype=np.float64).reshape(self.M, self.d)
        self.V = np.array(V, dtype=np.float64).reshape(self.M, self.d)
        self.score = np.array(score, dtype=np.float64).reshape(self.M)
        self.pos = np.array(pos, dtype=np.int64).reshape(self.M)
        self.t0 = int(t0)

    def step(self, q_g, k_new, v_new):
        """One chunk: attend, accumulate, evict, scatter.  Returns out [G, S, d]."""
        S = k_new.shape[0]
        t0 = self.t0
        valid = self.pos >= 0
        out, c_slots, c_new = attend_group(q_g, self.K, self.V, valid, k_new, v_new,
                                           1.0 / math.sqrt(self.d))
        # accumulate: running sum, no decay (pages define no normalisation)
        self.score[valid] += c_slots[valid]
        self.last_pre_scores = self.score.copy()
        self.last_c_slots, self.last_c_new = c_slots, c_new
        # evict: empty slots (a suffix, filled in slot order) are used first
        empties = [s for s in range(self.M) if self.pos[s] < 0]
        need = max(0, S - len(empties))
        if S > self.M:
            raise OracleShapeError(f"chunk of {S} tokens exceeds cache capacity {self.M}")
        self.last_eligible = (self.pos >= 0) & (self.pos < t0 - self.R)
        self.last_need = need
        if self.policy == "h2o":
            evicted = select_evictions(self.score, self.pos, t0, self.R, need)
        else:
            evicted = select_oldest(self.pos, t0, self.R, need)
        freed = sorted(evicted + empties[: S - need])
        # scatter: ascending freed slot <-> ascending new position
        for i, s in enumerate(freed):
            self.K[s] = k_new[i]
            self.V[s] = v_new[i]
            self.pos[s] = t0 + i
            self.score[s] = c_new[i]
        self.last_freed = np.array(freed, dtype=np.int64)
        self.t0 = t0 + S
        return out


class H2OOracle:
    """All (batch, KV head) caches of one layer; layouts as the library's:
    q, out [B, Hq, S, d]; k, v [B, Hkv, S, d]; query head g uses KV head g // G."""

    def __init__(self, M, R, Hq, Hkv, d, heads=None, policy="h2o"):
        if Hq % Hkv:
            raise ValueError("Hq must be a multiple of Hkv")
        self.policy = policy
        self.M, self.R, self.Hq, self.Hkv, self.d = int(M), int(R), int(Hq), int(Hkv), int(d)
        self.G = self.Hq // self.Hkv
        self.B = None
        self.t0 = 0
        self._only = None if heads is None else [tuple(x) for x in heads]
        self.heads = {}

    def _head_list(self):
        if self._only is not None:
            return self._only
        return [(b, h) for b in range(self.B) for h in range(self.Hkv)]

    def prefill(self, q, k, v):
        q, k, v = (np.asarray(x) for x in (q, k, v))
        B, Hq, P, d = q.shape
        if P > self.M:
            raise OracleShapeError(f"prefill of {P} tokens exceeds cache capacity {self.M}")
        self.B = B
        self.heads = {bh: H2OHeadOracle(self.M, self.R, self.G, self.d, self.policy)
                      for bh in self._head_list()}
        self.t0 = 0
        return self.step(q, k, v)

    def step(self, q, k, v):
        q, k, v = (np.asarray(x) for x in (q, k, v))
        B, Hq, S, d = q.shape
        out = np.full((B, Hq, S, d), np.nan, dtype=np.float64)
        for (b, h), st in self.heads.items():
            g0 = h * self.G
            out[b, g0:g0 + self.G] = st.step(q[b, g0:g0 + self.G], k[b, h], v[b, h])
        self.t0 += S
        return out

    def state(self):
        """(freed [B,Hkv,S], score [B,Hkv,M], pos [B,Hkv,M]) for the heads tracked."""
        return {bh: (st.last_freed, st.score.copy(), st.pos.copy()) for bh, st in self.heads.items()}
