"""Pins of the float64 oracle against facts fixed from outside it (CPU only).

Each pin is chosen so that a plausible slip in the oracle -- a dropped term, a
wrong sign or index, a transposed operand, an off-by-one window, a reversed
tie-break -- fails at least one of them; the mutation tests at the end plant such
slips in the oracle and check that a pin catches each.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle.h2o_oracle as ho
from oracle import H2OHeadOracle, H2OOracle, OracleShapeError, brute_stream, select_evictions

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
_ORIG_ATTEND = ho.attend_group


def _frac(s):
    return float(Fraction(s))


# --------------------------------------------------------------------------------------
# P1: the hand-worked 8-token example (exact fractions)
# --------------------------------------------------------------------------------------
def _eight_token_case():
    with open(os.path.join(GOLDEN, "eight_token_example.json")) as f:
        g = json.load(f)
    w = np.array(g["w"], dtype=np.float64)
    T = len(w)
    q = np.ones((1, 1, T, 1))
    k = np.log(w).reshape(1, 1, T, 1)
    v = np.array(g["v"], dtype=np.float64).reshape(1, 1, T, 1)
    return g, q, k, v


def check_eight_token_example():
    g, q, k, v = _eight_token_case()
    c = g["config"]
    orc = H2OOracle(c["M"], c["R"], c["Hq"], c["Hkv"], c["d"])
    P, S = c["prefill"], c["chunk"]
    outs = [orc.prefill(q[:, :, :P], k[:, :, :P], v[:, :, :P])]
    st = orc.heads[(0, 0)]
    np.testing.assert_allclose(st.pos, g["after_prefill"]["pos"])
    np.testing.assert_allclose(st.score, [_frac(s) for s in g["after_prefill"]["scores"]],
                               rtol=0, atol=1e-12)
    for name, t0 in (("chunk1", P), ("chunk2", P + S)):
        outs.append(orc.step(q[:, :, t0:t0 + S], k[:, :, t0:t0 + S], v[:, :, t0:t0 + S]))
        exp = g[name]
        np.testing.assert_allclose(st.last_pre_scores, [_frac(s) for s in exp["pre_evict_scores"]],
                                   rtol=0, atol=1e-12)
        assert st.last_freed.tolist() == exp["freed"]
        assert st.pos.tolist() == exp["pos"]
        np.testing.assert_allclose(st.score, [_frac(s) for s in exp["scores"]], rtol=0, atol=1e-12)
    got = np.concatenate([o[0, 0, :, 0] for o in outs])
    np.testing.assert_allclose(got, [_frac(s) for s in g["outputs"]], rtol=0, atol=1e-12)


def test_eight_token_example():
    check_eight_token_example()


def test_eight_token_example_brute_force():
    g, q, k, v = _eight_token_case()
    c = g["config"]
    res = brute_stream(q[0], k[0], v[0], c["M"], c["R"], c["prefill"], c["chunk"])
    np.testing.assert_allclose(res["outs"][0, :, 0], [_frac(s) for s in g["outputs"]], atol=1e-12)
    assert res["cached"][-1][0] == sorted(g["chunk2"]["pos"])
    want = dict(zip(g["chunk2"]["pos"], (_frac(s) for s in g["chunk2"]["scores"])))
    for p, s in res["scores"][-1][0].items():
        assert abs(s - want[p]) < 1e-12


# --------------------------------------------------------------------------------------
# P2: every chunk adds exactly S*G of mass per KV head (rows of a softmax sum to 1)
# --------------------------------------------------------------------------------------
def _rand_stream(rng, Hq, Hkv, T, d, B=1):
    q = rng.standard_normal((B, Hq, T, d)) * 0.5
    k = rng.standard_normal((B, Hkv, T, d)) * 0.5
    v = rng.standard_normal((B, Hkv, T, d)) * 0.5
    return q, k, v


def check_mass_invariant():
    rng = np.random.default_rng(1)
    Hq, Hkv, d, M, R, P, S, T = 6, 2, 8, 24, 4, 16, 8, 56
    q, k, v = _rand_stream(rng, Hq, Hkv, T, d, B=2)
    orc = H2OOracle(M, R, Hq, Hkv, d)
    G = Hq // Hkv
    orc.prefill(q[:, :, :P], k[:, :, :P], v[:, :, :P])
    for st in orc.heads.values():
        assert abs(st.last_c_slots.sum() + st.last_c_new.sum() - P * G) < 1e-9
    for t0 in range(P, T, S):
        orc.step(q[:, :, t0:t0 + S], k[:, :, t0:t0 + S], v[:, :, t0:t0 + S])
        for st in orc.heads.values():
            assert abs(st.last_c_slots.sum() + st.last_c_new.sum() - S * G) < 1e-9
            assert st.last_need == (0 if t0 == P else S)   # first chunk fills the empty slots


def test_mass_invariant():
    check_mass_invariant()


# --------------------------------------------------------------------------------------
# P3: a cache that never fills is exact causal attention (library SDPA, float64)
# --------------------------------------------------------------------------------------
def check_exact_attention_when_cache_never_fills(Hq=4, Hkv=2, d=16, P=24, S=8, T=64, B=2):
    rng = np.random.default_rng(2)
    q, k, v = _rand_stream(rng, Hq, Hkv, T, d, B=B)
    M = T + 5
    orc = H2OOracle(M, 3, Hq, Hkv, d)
    outs = [orc.prefill(q[:, :, :P], k[:, :, :P], v[:, :, :P])]
    for t0 in range(P, T, S):
        outs.append(orc.step(q[:, :, t0:t0 + S], k[:, :, t0:t0 + S], v[:, :, t0:t0 + S]))
    got = np.concatenate(outs, axis=2)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True,
                                                           enable_gqa=True).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # scores: column sums of the full causal softmax, summed over each group's heads
    G = Hq // Hkv
    logits = torch.einsum("bhid,bhjd->bhij", tq, tk.repeat_interleave(G, dim=1)) / math.sqrt(d)
    causal = torch.ones(T, T, dtype=torch.bool).tril()
    pw = torch.softmax(logits.masked_fill(~causal, float("-inf")), dim=-1)
    col = pw.sum(dim=2).reshape(B, Hkv, G, T).sum(dim=2).numpy()          # [B, Hkv, T]
    for (b, h), st in orc.heads.items():
        assert st.pos[:T].tolist() == list(range(T)) and (st.pos[T:] == -1).all()
        np.testing.assert_allclose(st.score[:T], col[b, h], rtol=0, atol=1e-10)


def test_exact_attention_when_cache_never_fills():
    check_exact_attention_when_cache_never_fills()


def test_exact_attention_ragged_chunks():
    check_exact_attention_when_cache_never_fills(Hq=3, Hkv=1, d=5, P=7, S=5, T=29, B=1)


# --------------------------------------------------------------------------------------
# P4: the slot oracle against the position-indexed brute force, with evictions
# --------------------------------------------------------------------------------------
def check_brute_force(seed=3, Hq=4, Hkv=2, d=4, M=12, R=3, P=8, S=4, T=32):
    rng = np.random.default_rng(seed)
    q, k, v = _rand_stream(rng, Hq, Hkv, T, d)
    k[0, :, ::5] *= 3.0                                  # a few louder keys: uneven scores
    res = brute_stream(q[0], k[0], v[0], M, R, P, S)
    orc = H2OOracle(M, R, Hq, Hkv, d)
    outs = [orc.prefill(q[:, :, :P], k[:, :, :P], v[:, :, :P])]
    bounds = [(t0, min(T, t0 + S)) for t0 in range(P, T, S)]
    for ci in range(len(bounds) + 1):
        if ci:
            t0, t1 = bounds[ci - 1]
            outs.append(orc.step(q[:, :, t0:t1], k[:, :, t0:t1], v[:, :, t0:t1]))
        for h in range(Hkv):
            st = orc.heads[(0, h)]
            assert sorted(st.pos[st.pos >= 0].tolist()) == res["cached"][ci][h]
            for s in np.nonzero(st.pos >= 0)[0]:
                assert abs(st.score[s] - res["scores"][ci][h][int(st.pos[s])]) < 1e-12
    np.testing.assert_allclose(np.concatenate(outs, axis=2)[0], res["outs"], atol=1e-12)


def test_brute_force_with_evictions():
    check_brute_force()


def test_brute_force_ragged_last_chunk():
    check_brute_force(seed=4, Hq=2, Hkv=1, d=3, M=9, R=2, P=5, S=3, T=21)


# --------------------------------------------------------------------------------------
# P5: selection against numpy's lexsort (scores with many exact ties)
# --------------------------------------------------------------------------------------
def check_select_vs_lexsort(trials=200):
    rng = np.random.default_rng(5)
    for _ in range(trials):
        M = int(rng.integers(1, 40))
        t0 = int(rng.integers(0, 100))
        R = int(rng.integers(0, 20))
        pos = rng.permutation(100)[:M].astype(np.int64)
        pos[rng.random(M) < 0.15] = -1
        score = rng.integers(0, 5, size=M) / 4.0            # exact ties
        elig = np.nonzero((pos >= 0) & (pos < t0 - R))[0]
        need = int(rng.integers(0, elig.size + 1))
        order = np.lexsort((pos[elig], score[elig]))         # primary score, then pos
        want = sorted(elig[order[:need]].tolist())
        assert ho.select_evictions(score, pos, t0, R, need) == want


def test_select_vs_lexsort():
    check_select_vs_lexsort()


def test_select_window_boundary():
    # pos == t0 - R is protected; pos == t0 - R - 1 is not
    score = np.array([0.0, 0.0])
    pos = np.array([6, 7])
    assert select_evictions(score, pos, t0=10, R=3, need=1) == [0]
    with pytest.raises(OracleShapeError):
        select_evictions(score, pos, t0=10, R=3, need=2)


# --------------------------------------------------------------------------------------
# Closed forms: uniform attention (q = 0) and duplicated query heads
# --------------------------------------------------------------------------------------
def test_uniform_attention_closed_form():
    Hq, Hkv, d, M, R, P, S = 2, 1, 4, 10, 2, 10, 4
    G = Hq // Hkv
    rng = np.random.default_rng(6)
    T = P + S
    q = np.zeros((1, Hq, T, d))
    k = rng.standard_normal((1, Hkv, T, d))
    v = rng.standard_normal((1, Hkv, T, d))
    orc = H2OOracle(M, R, Hq, Hkv, d)
    out = orc.prefill(q[:, :, :P], k[:, :, :P], v[:, :, :P])
    st = orc.heads[(0, 0)]
    tail = [sum(1.0 / (i + 1) for i in range(j, P)) for j in range(P)]   # harmonic tails
    np.testing.assert_allclose(st.score, G * np.array(tail), atol=1e-12)
    for i in range(P):
        np.testing.assert_allclose(out[0, 0, i], v[0, 0, :i + 1].mean(axis=0), atol=1e-12)
    before = st.score.copy()
    out = orc.step(q[:, :, P:], k[:, :, P:], v[:, :, P:])
    inc = G * sum(1.0 / (M + i + 1) for i in range(S))
    np.testing.assert_allclose(st.last_pre_scores, before + inc, atol=1e-12)
    # lowest pre-eviction scores among pos < P - R are the latest eligible tokens
    assert st.last_freed.tolist() == list(range(P - R - S, P - R))
    for i in range(S):
        want = G * sum(1.0 / (M + r + 1) for r in range(i, S))
        assert abs(st.score[P - R - S + i] - want) < 1e-12


def test_duplicated_query_heads_double_the_scores():
    rng = np.random.default_rng(7)
    d, M, R, P, S, T = 4, 10, 2, 8, 4, 24
    q1, k, v = _rand_stream(rng, 1, 1, T, d)
    q2 = np.concatenate([q1, q1], axis=1)
    a, b = H2OOracle(M, R, 1, 1, d), H2OOracle(M, R, 2, 1, d)
    oa, ob = a.prefill(q1[:, :, :P], k[:, :, :P], v[:, :, :P]), b.prefill(q2[:, :, :P], k[:, :, :P], v[:, :, :P])
    for t0 in range(P, T, S):
        oa = a.step(q1[:, :, t0:t0 + S], k[:, :, t0:t0 + S], v[:, :, t0:t0 + S])
        ob = b.step(q2[:, :, t0:t0 + S], k[:, :, t0:t0 + S], v[:, :, t0:t0 + S])
        np.testing.assert_allclose(ob[:, 1], oa[:, 0], atol=1e-12)
        sa, sb = a.heads[(0, 0)], b.heads[(0, 0)]
        np.testing.assert_allclose(sb.score, 2 * sa.score, atol=1e-12)
        assert sb.pos.tolist() == sa.pos.tolist()


def test_shape_errors():
    orc = H2OOracle(4, 1, 1, 1, 2)
    x = np.zeros((1, 1, 5, 2))
    with pytest.raises(OracleShapeError):
        orc.prefill(x, x, x)
    st = H2OHeadOracle(M=4, R=3, G=1, d=2)
    st.step(np.zeros((1, 4, 2)), np.zeros((4, 2)), np.zeros((4, 2)))
    with pytest.raises(OracleShapeError):     # only pos 0 is older than the window
        st.step(np.zeros((1, 2, 2)), np.zeros((2, 2)), np.zeros((2, 2)))


# --------------------------------------------------------------------------------------
# Mutation tests: plant a plausible slip in the oracle, check that a pin catches it
# --------------------------------------------------------------------------------------
def _attend_causal_strict(q_g, k_slots, v_slots, slot_valid, k_new, v_new, scale, row_block=512):
    # slip: a chunk row does not see its own key (j < i instead of j <= i)
    G, S, d = q_g.shape
    out = np.zeros((G, S, d))
    valid_idx = np.nonzero(slot_valid)[0]
    keys = np.concatenate([k_slots[valid_idx], k_new])
    vals = np.concatenate([v_slots[valid_idx], v_new])
    n_c = valid_idx.size
    col = np.zeros(n_c + S)
    for g in range(G):
        for i in range(S):
            n = n_c + max(i, 1)
            lg = keys[:n] @ q_g[g, i] * scale
            p = np.exp(lg - lg.max())
            p /= p.sum()
            out[g, i] = p @ vals[:n]
            col[:n] += p
    cs = np.zeros(k_slots.shape[0])
    cs[valid_idx] = col[:n_c]
    return out, cs, col[n_c:]


def _select_newest_first(score, pos, t0, R, need):
    # slip: ties broken toward the newer token
    elig = [s for s in range(len(score)) if 0 <= pos[s] < t0 - R]
    if need > len(elig):
        raise OracleShapeError("short")
    return sorted(sorted(elig, key=lambda s: (score[s], -pos[s]))[:need])


def _select_window_after_chunk(score, pos, t0, R, need):
    # slip: the window is counted one token later (pos <= t0 - R eligible)
    elig = [s for s in range(len(score)) if 0 <= pos[s] <= t0 - R]
    if need > len(elig):
        raise OracleShapeError("short")
    return sorted(sorted(elig, key=lambda s: (score[s], pos[s]))[:need])


def _attend_row_sums(q_g, k_slots, v_slots, slot_valid, k_new, v_new, scale, row_block=512):
    # slip: transposed reduction -- mass spread evenly instead of per column
    out, cs, cn = _ORIG_ATTEND(q_g, k_slots, v_slots, slot_valid, k_new, v_new, scale)
    total = cs.sum() + cn.sum()
    n = int(np.count_nonzero(slot_valid)) + cn.size
    cs = np.where(slot_valid, total / n, 0.0)
    return out, cs, np.full(cn.size, total / n)


def _attend_scale_inv_d(q_g, k_slots, v_slots, slot_valid, k_new, v_new, scale, row_block=512):
    # slip: 1/d instead of 1/sqrt(d)
    d = q_g.shape[-1]
    return _ORIG_ATTEND(q_g, k_slots, v_slots, slot_valid, k_new, v_new, 1.0 / d)


@pytest.mark.parametrize("target,mutant", [
    ("attend_group", _attend_causal_strict),
    ("attend_group", _attend_row_sums),
    ("attend_group", _attend_scale_inv_d),
    ("select_evictions", _select_newest_first),
    ("select_evictions", _select_window_after_chunk),
])
def test_pins_catch_planted_slips(monkeypatch, target, mutant):
    monkeypatch.setattr(ho, target, mutant)
    pins = [check_eight_token_example, check_mass_invariant,
            check_exact_attention_when_cache_never_fills, check_brute_force,
            lambda: check_select_vs_lexsort(50)]
    caught = 0
    for pin in pins:
        try:
            pin()
        except (AssertionError, OracleShapeError):
            caught += 1
    assert caught >= 1, f"no pin caught the planted slip in {target}"


# --------------------------------------------------------------------------------------
# The recency-only policy (lr): closed form and windowed attention from a library routine
# --------------------------------------------------------------------------------------
def _lr_stream(select=None, seed=7, Hq=4, Hkv=2, d=8, M=24, R=5, P=16, S=6, T=16 + 6 * 8 + 3, B=2):
    rng = np.random.default_rng(seed)
    q, k, v = _rand_stream(rng, Hq, Hkv, T, d, B=B)
    orc = H2OOracle(M, R, Hq, Hkv, d, policy="lr")
    bounds = [(0, P)] + [(t, min(T, t + S)) for t in range(P, T, S)]
    outs, cached = [], []
    for i, (a, b) in enumerate(bounds):
        x = (q[:, :, a:b], k[:, :, a:b], v[:, :, a:b])
        outs.append(orc.prefill(*x) if i == 0 else orc.step(*x))
        cached.append({bh: sorted(int(p) for p in st.pos if p >= 0) for bh, st in orc.heads.items()})
    return q, k, v, orc, bounds, np.concatenate(outs, axis=2), cached


def check_lr_holds_the_most_recent_tokens():
    M = 24
    *_, bounds, _, cached = _lr_stream(M=M)
    for (a, b), c in zip(bounds, cached):
        for heads in c.values():
            assert heads == list(range(max(0, b - M), b)), (b, heads)


def test_lr_holds_the_most_recent_tokens():
    # closed form: with M - R >= S the oldest tokens are always evictable, so after
    # every chunk the cache holds exactly the last M positions
    check_lr_holds_the_most_recent_tokens()


def test_lr_outputs_equal_chunked_window_attention():
    # the query at t0 + i of a chunk starting at t0 sees positions
    # [max(0, t0 - M), t0 + i]: library SDPA with that explicit mask, float64
    M, Hq, Hkv, d = 24, 4, 2, 8
    q, k, v, orc, bounds, got, _ = _lr_stream(M=M, Hq=Hq, Hkv=Hkv, d=d)
    T = q.shape[2]
    allow = torch.zeros(T, T, dtype=torch.bool)
    for a, b in bounds:
        for t in range(a, b):
            allow[t, max(0, a - M):t + 1] = True
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=allow,
                                                           enable_gqa=True).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # the summed weights still carry S * G of mass per KV head and chunk
    for st in orc.heads.values():
        S = bounds[-1][1] - bounds[-1][0]
        assert abs(st.last_c_slots.sum() + st.last_c_new.sum() - S * (Hq // Hkv)) < 1e-9


def test_lr_pin_catches_a_newest_first_slip(monkeypatch):
    # a plausible slip -- evicting the newest eligible tokens -- fails the closed form
    def newest(pos, t0, R, need):
        elig = [s for s in range(len(pos)) if 0 <= pos[s] < t0 - R]
        return sorted(sorted(elig, key=lambda s: -int(pos[s]))[:need])
    monkeypatch.setattr(ho, "select_oldest", newest)
    with pytest.raises(AssertionError):
        check_lr_holds_the_most_recent_tokens()
