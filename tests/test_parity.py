"""GPU path vs the float64 oracle, through the C ABI (needs a B200).

Every chunk of a seeded stream runs on the GPU (prefill, then steps) and in the
oracle on the same input values; outputs, scores, evictions, slot -> position
maps and the cache's K/V bytes are compared with the tolerances of
tests/parity_util.py.  Small configurations run the oracle on every head and
every chunk; the full-size workloads run it on sampled (batch, KV head) caches
-- either along the whole stream, or on sampled chunks after loading the GPU's
state into the oracle.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest
import torch

from oracle import H2OHeadOracle, H2OOracle, select_evictions
from tests.parity_util import (annotate_boundary, check_evictions, check_outputs, check_scores,
                               check_tie_state, to64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h2o(cuda_ok):
    import h2o_kv_cache_b200 as m
    return m


def _cfg(base, **kw):
    from h2o_kv_cache_b200.workload import CONFIGS
    return dataclasses.replace(CONFIGS[base] if isinstance(base, int) else base, **kw)


def _sync_head(st, kc, vc, scores, pos, b, h, t0):
    st.load_state(to64(kc[b, h]), to64(vc[b, h]), scores[b, h], pos[b, h], t0)


def run_stream(h2o, cfg, heads=None, layer=0, T=None, oracle_chunks=None, kv_check=True,
               policy="h2o"):
    """Returns a summary dict.  oracle_chunks=None: the oracle follows the whole
    stream; otherwise only the listed chunk indices are checked, each after
    loading the GPU's pre-step state into the oracle."""
    from h2o_kv_cache_b200.workload import gen_batch, split_chunks
    T = cfg.T if T is None else T
    Q, K, V = gen_batch(cfg, layer, device="cuda", T=T)
    bounds = [(a, b) for a, b in cfg.bounds() if a < T]
    bounds[-1] = (bounds[-1][0], min(bounds[-1][1], T))
    chunks = split_chunks(Q, K, V, bounds)
    cache = h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype, policy=policy)
    G = cfg.G
    if heads is None:
        heads = [(b, h) for b in range(cfg.B) for h in range(cfg.Hkv)]
    orc = {bh: H2OHeadOracle(cfg.M, cfg.R, G, cfg.d, policy) for bh in heads}
    Kn, Vn = to64(K), to64(V)
    summary = {"chunks": 0, "ties": 0, "max_abs": 0.0, "rel_norm": 0.0, "score_rel": 0.0}
    for ci, (q, k, v) in enumerate(chunks):
        t0 = bounds[ci][0]
        follow = oracle_chunks is None or ci in oracle_chunks
        if follow and oracle_chunks is not None and ci > 0:
            _, sc0, ps0 = cache.read_state()
            kc0, vc0 = cache.read_kv()
            sc0, ps0 = sc0.cpu().numpy(), ps0.cpu().numpy()
            for (b, h), st in orc.items():
                _sync_head(st, kc0, vc0, sc0, ps0, b, h, t0)
        pos_before = {bh: st.pos.copy() for bh, st in orc.items()}
        out = cache.prefill(q, k, v) if ci == 0 else cache.step(q, k, v)
        torch.cuda.synchronize()
        if not follow:
            continue
        slots, scores, pos = (x.cpu().numpy() for x in cache.read_state())
        d_slots, d_evicted = (x.cpu().numpy() for x in cache.read_delta())
        assert np.array_equal(d_slots, slots)
        out64 = to64(out)
        qn = to64(q)
        kn_, vn_ = to64(k), to64(v)
        kc = vc = None
        for (b, h), st in orc.items():
            gq = slice(h * G, (h + 1) * G)
            ref = st.step(qn[b, gq], kn_[b, h], vn_[b, h])
            where = f"{cfg.name} chunk {ci} (b={b}, h={h})"
            r = check_outputs(out64[b, gq], ref, cfg.dtype, where)
            summary["max_abs"] = max(summary["max_abs"], r["max_abs"])
            summary["rel_norm"] = max(summary["rel_norm"], r["rel_norm"])
            annotate_boundary(st, pos_before[(b, h)])
            if policy == "lr":   # positions are unique: the evicted set is fixed, no ties
                assert np.array_equal(slots[b, h], st.last_freed), f"{where}: filled slots differ"
            status = check_evictions(st, slots[b, h], where)
            if status == "exact":
                assert np.array_equal(pos[b, h], st.pos), f"{where}: slot -> position map differs"
                # the buffer delta: each filled slot's previous token (-1: it was empty)
                assert np.array_equal(d_evicted[b, h], pos_before[(b, h)][slots[b, h]]), \
                    f"{where}: evicted positions differ"
                summary["score_rel"] = max(summary["score_rel"],
                                           check_scores(scores[b, h], st.score, st.pos >= 0, where))
            else:
                summary["ties"] += 1
                check_tie_state(slots[b, h], pos[b, h], pos_before[(b, h)], t0, where)
                assert np.array_equal(d_evicted[b, h], pos_before[(b, h)][slots[b, h]]), \
                    f"{where}: evicted positions differ"
                # compare by position on the tokens both kept, then adopt the GPU state
                gmap = {int(p): s for p, s in zip(pos[b, h], scores[b, h]) if p >= 0}
                omap = {int(p): s for p, s in zip(st.pos, st.score) if p >= 0}
                common = sorted(set(gmap) & set(omap))
                check_scores(np.array([gmap[p] for p in common]), np.array([omap[p] for p in common]),
                             np.ones(len(common), bool), where)
                if kc is None:
                    kc, vc = cache.read_kv()
                _sync_head(st, kc, vc, scores, pos, b, h, t0 + (bounds[ci][1] - bounds[ci][0]))
            if kv_check:
                if kc is None:
                    kc, vc = cache.read_kv()
                valid = pos[b, h] >= 0
                p = pos[b, h][valid]
                assert torch.equal(kc[b, h][torch.from_numpy(valid).cuda()], K[b, h, torch.from_numpy(p).long().cuda()]), f"{where}: cached K rows differ from the stream"
                assert torch.equal(vc[b, h][torch.from_numpy(valid).cuda()], V[b, h, torch.from_numpy(p).long().cuda()]), f"{where}: cached V rows differ from the stream"
        summary["chunks"] += 1
    info = cache.info()
    assert info["t0"] == bounds[-1][1]
    cache.close()
    return summary


# --------------------------------------------------------------------------------------
# Small configurations: every head, every chunk
# --------------------------------------------------------------------------------------
def test_tiny_fp32_full_stream(h2o):
    s = run_stream(h2o, _cfg(0))
    assert s["chunks"] == 5


def test_exact_attention_when_cache_never_fills(h2o):
    cfg = _cfg(0, M=384, name="tiny-fp32-never-full")
    s = run_stream(h2o, cfg)
    assert s["ties"] == 0


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.float32, 128),
                                     (torch.bfloat16, 64), (torch.bfloat16, 128)])
def test_ragged_shapes(h2o, dtype, d):
    # ragged prefill (partly full cache), ragged chunks, a ragged last chunk, B > 1
    cfg = _cfg(0, name=f"ragged-{dtype}-{d}", B=2, Hq=6, Hkv=2, d=d, M=300, R=17, T=100 + 37 * 7 + 11,
               P=100, S=37, dtype=dtype, planted=0.02)
    run_stream(h2o, cfg)


def test_large_gqa_group_and_long_tile_rows(h2o):
    cfg = _cfg(0, name="gqa8-bf16", B=1, Hq=8, Hkv=1, d=128, M=520, R=40, T=520 + 3 * 260, P=520,
               S=260, dtype=torch.bfloat16, planted=0.01)
    run_stream(h2o, cfg)


def test_single_token_steps_and_single_token_prefill(h2o):
    cfg = _cfg(0, name="decode-like", M=40, R=4, T=1 + 70, P=1, S=1, planted=0.0)
    run_stream(h2o, cfg)
    cfg = _cfg(0, name="decode-bf16", M=72, R=5, T=72 + 30, P=72, S=1, dtype=torch.bfloat16, d=128)
    run_stream(h2o, cfg)


def test_window_just_below_capacity(h2o):
    # R = M - S: exactly `need` slots are evictable at every step
    cfg = _cfg(0, name="tight-window", M=96, R=64, T=96 + 32 * 5, P=96, S=32)
    run_stream(h2o, cfg)


@pytest.mark.parametrize("split", ["2", "4", "8"])
def test_keys_split_across_a_cluster(h2o, monkeypatch, split):
    # each unit's keys shared by `split` CTAs: exchanged row statistics and summed partial O
    monkeypatch.setenv("H2O_ATTN_MODE", "fused")
    monkeypatch.setenv("H2O_ATTN_SPLIT", split)
    cfg = _cfg(1)
    s = run_stream(h2o, cfg, heads=[(0, 0), (0, 5)], T=cfg.P + 2 * cfg.S)
    assert s["chunks"] == 3


def test_split_with_odd_tile_counts(h2o, monkeypatch):
    # 8 cache tiles + 1-2 chunk tiles per unit: the last CTA of a cluster gets an odd tile
    monkeypatch.setenv("H2O_ATTN_MODE", "fused")
    monkeypatch.setenv("H2O_ATTN_SPLIT", "4")
    cfg = _cfg(0, name="split-odd", B=1, Hq=6, Hkv=2, d=128, M=1000, R=90, T=1000 + 4 * 200 + 77,
               P=1000, S=200, dtype=torch.bfloat16, planted=0.02)
    run_stream(h2o, cfg)


@pytest.mark.parametrize("case", ["ragged", "gqa8", "odd-tiles", "decode", "m2k-fused"])
def test_stream_and_fused_paths(h2o, monkeypatch, case):
    # the two tensor-core paths on shapes that stress the stream partition: ragged
    # prefill and chunks, B > 1, an odd number of query heads per KV head (no head B
    # in the last pair), units whose last pair has one tile, single-token steps; and
    # the one-kernel path at the size where the stream path is the default
    mode = "fused" if case == "m2k-fused" else "stream"
    monkeypatch.setenv("H2O_ATTN_MODE", mode)
    bf = dict(dtype=torch.bfloat16, d=128)
    cfgs = {
        "ragged": _cfg(0, name="stream-ragged", B=2, Hq=6, Hkv=2, M=300, R=17, T=100 + 37 * 7 + 11,
                       P=100, S=37, planted=0.02, **bf),
        "gqa8": _cfg(0, name="stream-gqa8", B=1, Hq=8, Hkv=1, M=520, R=40, T=520 + 3 * 260, P=520,
                     S=260, planted=0.01, **bf),
        "odd-tiles": _cfg(0, name="stream-odd", B=1, Hq=6, Hkv=2, M=1000, R=90, T=1000 + 4 * 200 + 77,
                          P=1000, S=200, planted=0.02, **bf),
        "decode": _cfg(0, name="stream-decode", M=72, R=5, T=72 + 30, P=72, S=1, **bf),
        "m2k-fused": _cfg(1),
    }
    cfg = cfgs[case]
    T = cfg.P + 3 * cfg.S if case == "m2k-fused" else None
    s = run_stream(h2o, cfg, T=T, heads=[(0, 1), (0, 6)] if case == "m2k-fused" else None)
    assert s["chunks"] >= 2


@pytest.mark.parametrize("S,dtype,d", [(1, torch.bfloat16, 128), (2, torch.bfloat16, 128),
                                       (4, torch.bfloat16, 64), (1, torch.float32, 64),
                                       (3, torch.float32, 128)])
def test_decode_kernel_small_chunks(h2o, S, dtype, d):
    # G * S <= 16 rows per KV head: the key-split FMA kernel (G = 4 here), a ragged
    # cache that fills and then evicts every step
    cfg = _cfg(0, name=f"decode-{S}-{d}", B=2, Hq=8, Hkv=2, d=d, M=150, R=9, P=100, S=S,
               T=100 + 60 * S + (S > 1), dtype=dtype, planted=0.02)
    s = run_stream(h2o, cfg)
    assert s["chunks"] >= 60


def test_decode_kernel_m2k_and_m32k(h2o):
    # decode steps on the benchmark caches: every key split over a cluster
    cfg = _cfg(1, name="m2k-decode", S=1)
    run_stream(h2o, cfg, heads=[(0, 0), (0, 7)], T=cfg.P + 40)
    cfg = _cfg(3, name="m32k-decode", S=1)
    run_stream(h2o, cfg, heads=[(0, 3)], T=cfg.P + 6, kv_check=False)
    # 16 rows per KV head (S = 4, G = 4) on the 32k-slot cache: the scores do not
    # fit the decode kernel's shared memory, so the step takes the tensor-core path
    cfg = _cfg(3, name="m32k-s4", S=4)
    run_stream(h2o, cfg, heads=[(0, 5)], T=cfg.P + 8, kv_check=False)


def test_small_chunks_s128(h2o):
    # S = 128: 16 units for 148 SMs, so the kernel splits each unit's keys
    cfg = _cfg(1, name="m2k-s128", S=128)
    s = run_stream(h2o, cfg, T=cfg.P + 6 * 128)
    assert s["chunks"] == 7


# --------------------------------------------------------------------------------------
# The benchmark workloads at full size
# --------------------------------------------------------------------------------------
def test_m2k_s1k_full_stream(h2o):
    s = run_stream(h2o, _cfg(1))
    assert s["chunks"] == 15


def test_m16k_s1k_sampled_head_full_stream(h2o):
    run_stream(h2o, _cfg(2), heads=[(0, 3)], kv_check=False)


def test_m32k_s2k_sampled_chunks(h2o):
    run_stream(h2o, _cfg(3), heads=[(0, 5)], oracle_chunks={1, 2, 48})


def test_b4_layers_sampled_heads(h2o):
    cfg = _cfg(4)
    run_stream(h2o, cfg, heads=[(2, 6)], layer=0, kv_check=False)
    run_stream(h2o, cfg, heads=[(1, 1)], layer=27, oracle_chunks={1, 24}, kv_check=False)


# --------------------------------------------------------------------------------------
# Prefill mass invariant at full size, errors, host pointers, standalone selection
# --------------------------------------------------------------------------------------
def test_prefill_mass_invariant_full_size(h2o):
    from h2o_kv_cache_b200.workload import gen_batch
    cfg = _cfg(3)
    Q, K, V = gen_batch(cfg, 0, device="cuda", T=cfg.P)
    cache = h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype)
    cache.prefill(Q, K, V)
    _, scores, pos = cache.read_state()
    tot = scores.double().sum(dim=2)
    torch.testing.assert_close(tot, torch.full_like(tot, cfg.P * cfg.G), rtol=1e-4, atol=0)
    assert torch.equal(pos[0, 0], torch.arange(cfg.P, dtype=torch.int32, device="cuda"))
    cache.close()


def test_shape_error_leaves_state_intact(h2o):
    from h2o_kv_cache_b200.workload import gen_batch
    cfg = _cfg(0, M=64, R=60, T=64 + 8, P=64, S=8)
    Q, K, V = gen_batch(cfg, 0, device="cuda")
    cache = h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype)
    cache.prefill(Q[:, :, :64].contiguous(), K[:, :, :64].contiguous(), V[:, :, :64].contiguous())
    before = [x.clone() for x in cache.read_state()[1:]]
    with pytest.raises(h2o.H2OError) as ei:    # 64 valid, min(R, t0) = 60 protected, need 8
        cache.step(Q[:, :, 64:].contiguous(), K[:, :, 64:].contiguous(), V[:, :, 64:].contiguous())
    assert ei.value.status == -2
    after = cache.read_state()[1:]
    assert all(torch.equal(a, b) for a, b in zip(before, after))
    assert cache.info()["t0"] == 64
    cache.close()


@pytest.mark.parametrize("mode", ["fused", "stream"])
def test_bounded_wait_timeout_is_reported_and_context_stays_usable(h2o, monkeypatch, mode):
    # a wait on a barrier that nothing completes runs out (1 ms); every role of the
    # kernel leaves through its abort path, the step reports H2O_ETIMEOUT, and the
    # device context keeps working.  "stream": the hook sits in the second of the
    # two stream-partitioned kernels (four softmax warpgroups, per-piece barriers).
    from h2o_kv_cache_b200.workload import gen_batch, split_chunks
    monkeypatch.setenv("H2O_ATTN_MODE", mode)
    cfg = _cfg(0, dtype=torch.bfloat16, d=128)
    Q, K, V = gen_batch(cfg, 0, device="cuda")
    chunks = split_chunks(Q, K, V, cfg.bounds())
    cache = h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype)
    cache.prefill(*chunks[0])
    monkeypatch.setenv("H2O_INJECT_TIMEOUT", "1")
    monkeypatch.setenv("H2O_SYNC_CHECK", "1")
    with pytest.raises(h2o.H2OError) as ei:
        cache.step(*chunks[1])
    assert ei.value.status == -6, ei.value
    cache.close()
    monkeypatch.delenv("H2O_INJECT_TIMEOUT")
    monkeypatch.delenv("H2O_SYNC_CHECK")
    s = run_stream(h2o, cfg)
    assert s["chunks"] == 5


def test_host_buffers_match_device_buffers(h2o):
    from h2o_kv_cache_b200.workload import gen_batch, split_chunks
    cfg = _cfg(0, dtype=torch.bfloat16, d=128)
    Q, K, V = gen_batch(cfg, 0, device="cuda")
    chunks = split_chunks(Q, K, V, cfg.bounds())
    a = h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype)
    b = h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype)
    for ci, (q, k, v) in enumerate(chunks):
        pin = ci % 2 == 0
        hq, hk, hv = (x.cpu().pin_memory() if pin else x.cpu() for x in (q, k, v))
        hout = torch.empty_like(hq).pin_memory() if pin else torch.empty_like(hq)
        oa = a.prefill(q, k, v) if ci == 0 else a.step(q, k, v)
        ob = b.prefill(hq, hk, hv, out=hout) if ci == 0 else b.step(hq, hk, hv, out=hout)
        torch.cuda.synchronize()
        assert torch.equal(oa.cpu(), ob)
    for x, y in zip(a.read_state(), b.read_state()):
        assert torch.equal(x, y)
    a.close()
    b.close()


@pytest.mark.parametrize("stage", ["1", "0"])
@pytest.mark.parametrize("base,kw,T", [
    (0, {}, None),
    (0, {"dtype": torch.bfloat16, "d": 128, "M": 301, "R": 45, "P": 203, "S": 37}, 203 + 6 * 37 + 11),
    (1, {}, 2048 + 3 * 1024),
])
def test_fused_tail_matches_split_kernels(h2o, monkeypatch, base, kw, T, stage):
    """The fused cluster tail and the three separate kernels accumulate the
    summed weights the same way, so outputs, state and cache agree bit for bit;
    the fused kernel with its chunk rows staged in shared memory, and without
    (H2O_TAIL_STAGE=0: the register path that rows too large to stage take)."""
    from h2o_kv_cache_b200.workload import gen_batch, split_chunks
    monkeypatch.setenv("H2O_TAIL_STAGE", stage)
    cfg = _cfg(base, **kw)
    T = cfg.T if T is None else T
    Q, K, V = gen_batch(cfg, 0, device="cuda", T=T)
    bounds = [(a, b) for a, b in cfg.bounds() if a < T]
    bounds[-1] = (bounds[-1][0], min(bounds[-1][1], T))
    chunks = split_chunks(Q, K, V, bounds)
    fused = h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype)
    monkeypatch.setenv("H2O_SPLIT_TAIL", "1")
    split = h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype)
    for ci, (q, k, v) in enumerate(chunks):
        if ci == 0:
            monkeypatch.delenv("H2O_SPLIT_TAIL")
            of = fused.prefill(q, k, v)
            monkeypatch.setenv("H2O_SPLIT_TAIL", "1")
            os_ = split.prefill(q, k, v)
        else:
            monkeypatch.delenv("H2O_SPLIT_TAIL")
            of = fused.step(q, k, v)
            monkeypatch.setenv("H2O_SPLIT_TAIL", "1")
            os_ = split.step(q, k, v)
        assert split.info()["launches"] - fused.info()["launches"] == 2
        assert torch.equal(of, os_), f"chunk {ci}: outputs differ"
        for x, y in zip(fused.read_state() + fused.read_delta(), split.read_state() + split.read_delta()):
            assert torch.equal(x, y), f"chunk {ci}: state differs"
    for x, y in zip(fused.read_kv(), split.read_kv()):
        assert torch.equal(x, y)
    fused.close()
    split.close()


def test_fused_tail_every_cluster_size(h2o, monkeypatch):
    """The fused tail at cluster sizes 1 to 16 (H2O_TAIL_CS), powers of two or
    not, agrees bit for bit with the three separate kernels: per-CTA slot and
    chunk-row ranges that do not divide M and S, histogram bins owned by rank
    t mod cs, the per-rank counts of the ordered compaction."""
    from h2o_kv_cache_b200.workload import gen_batch, split_chunks
    cfg = _cfg(0, dtype=torch.bfloat16, d=128, B=1, Hq=8, Hkv=4, M=1000, R=64, P=1000, S=96,
               T=1000 + 4 * 96 + 17)
    Q, K, V = gen_batch(cfg, 0, device="cuda")
    chunks = split_chunks(Q, K, V, cfg.bounds())
    monkeypatch.setenv("H2O_SPLIT_TAIL", "1")
    ref = h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype)
    want = [ref.prefill(*chunks[0])] + [ref.step(*c) for c in chunks[1:]]
    torch.cuda.synchronize()
    want_state = [x.clone() for x in ref.read_state() + ref.read_delta() + ref.read_kv()]
    ref.close()
    monkeypatch.delenv("H2O_SPLIT_TAIL")
    for cs in (1, 2, 3, 5, 7, 10, 13, 16):
        monkeypatch.setenv("H2O_TAIL_CS", str(cs))
        c = h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype)
        got = [c.prefill(*chunks[0])] + [c.step(*ch) for ch in chunks[1:]]
        torch.cuda.synchronize()
        for ci, (a, b) in enumerate(zip(got, want)):
            assert torch.equal(a, b), f"clusters of {cs}, chunk {ci}: outputs differ"
        for x, y in zip(c.read_state() + c.read_delta() + c.read_kv(), want_state):
            assert torch.equal(x, y), f"clusters of {cs}: state differs"
        c.close()


def test_standalone_select_with_ties(h2o):
    rng = np.random.default_rng(11)
    for trial in range(12):
        n, M = 3, int(rng.integers(8, 5000))
        t0 = 10 * M
        R = int(rng.integers(0, M // 2))
        pos = np.stack([rng.permutation(t0)[:M] for _ in range(n)]).astype(np.int32)
        pos[rng.random((n, M)) < 0.05] = -1
        if trial % 3 == 0:
            scores = rng.integers(0, 4, size=(n, M)).astype(np.float32) / 8   # heavy ties
        elif trial % 3 == 1:
            scores = np.zeros((n, M), np.float32)                             # all tied
        else:
            scores = rng.random((n, M)).astype(np.float32)
        elig = (pos >= 0) & (pos < t0 - R)
        need = int(min(elig.sum(axis=1).min(), rng.integers(1, M)))
        if need == 0:
            continue
        ev = h2o.select(torch.from_numpy(scores).cuda(), torch.from_numpy(pos).cuda(), t0, R, need)
        for i in range(n):
            want = select_evictions(scores[i].astype(np.float64), pos[i], t0, R, need)
            assert ev[i].cpu().tolist() == want


def test_standalone_select_reports_too_few_eligible(h2o):
    scores = torch.zeros(1, 16, device="cuda")
    pos = torch.arange(16, dtype=torch.int32, device="cuda")[None]
    with pytest.raises(h2o.H2OError) as ei:
        h2o.select(scores, pos, t0=16, R=12, need=5)     # only pos 0..3 are eligible
    assert ei.value.status == -2


@pytest.mark.parametrize("kind", ["alloc", "launch"])
def test_host_fault_injection(h2o, monkeypatch, kind):
    # faults made on the host (H2O_FAULT): an allocation that fails at prefill,
    # a launch that fails at a step.  Each call reports its status and a message,
    # the handle can be destroyed, and a fresh handle runs the stream at parity.
    from h2o_kv_cache_b200.workload import gen_batch, split_chunks
    cfg = _cfg(0, dtype=torch.bfloat16, d=128)
    Q, K, V = gen_batch(cfg, 0, device="cuda")
    chunks = split_chunks(Q, K, V, cfg.bounds())
    cache = h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype)
    if kind == "alloc":
        monkeypatch.setenv("H2O_FAULT", "alloc")
        with pytest.raises(h2o.H2OError) as ei:
            cache.prefill(*chunks[0])
        assert ei.value.status == -4 and "alloc" in str(ei.value)
        monkeypatch.delenv("H2O_FAULT")
        cache.prefill(*chunks[0])           # the failed prefill left nothing behind
        assert cache.info()["t0"] == cfg.P
    else:
        cache.prefill(*chunks[0])
        monkeypatch.setenv("H2O_FAULT", "launch")
        with pytest.raises(h2o.H2OError) as ei:
            cache.step(*chunks[1])
        assert ei.value.status == -5 and "launch" in str(ei.value)
        assert cache.info()["t0"] == cfg.P   # the failed step did not advance
        monkeypatch.delenv("H2O_FAULT")
    cache.close()
    s = run_stream(h2o, cfg)
    assert s["chunks"] == 5


def _layer_streams(cfg, layers, T):
    from h2o_kv_cache_b200.workload import gen_batch, split_chunks
    bounds = [(a, b) for a, b in cfg.bounds() if a < T]
    out = []
    for layer in layers:
        Q, K, V = gen_batch(cfg, layer, device="cuda", T=T)
        out.append(split_chunks(Q, K, V, bounds))
    return out, bounds


@pytest.mark.parametrize("case", ["b4-3layers", "tiny-bf16-35layers", "mixed-fp32",
                                  "10layers-640caches"])
def test_step_layers_matches_single_steps(h2o, monkeypatch, case):
    """h2o_step_layers gives, bit for bit, what one h2o_step per layer gives: one
    grid for all layers' attention and one for all tails (b4: three layers of the
    28-layer workload; 35 small layers: two groups of at most 32), or per-layer
    launches when the path is not the one-kernel tensor-core one (fp32).  Keys
    are not split across CTAs here: a grid of one layer may split them where a
    grid of many layers does not, and a split adds partial outputs in another
    order (the summed weights are exact integers either way)."""
    monkeypatch.setenv("H2O_ATTN_SPLIT", "1")
    if case == "b4-3layers":
        cfg, n, T = _cfg(4), 3, None
        T = cfg.P + 3 * cfg.S
    elif case == "tiny-bf16-35layers":
        cfg, n = _cfg(0, dtype=torch.bfloat16, d=128, name="tiny-bf16"), 35
        T = cfg.T
    elif case == "mixed-fp32":
        cfg, n = _cfg(0), 3
        T = cfg.T
    else:
        # 10 layers x 64 caches: at least two waves of caches, so the grouped tail
        # runs one CTA per cache and moves the chunk rows with bulk copies
        cfg = _cfg(0, name="grouped-bulk-tail", B=8, Hq=16, Hkv=8, d=128, M=2048, R=128,
                   P=2048, S=256, T=2048 + 3 * 256, dtype=torch.bfloat16, planted=0.01)
        n, T = 10, cfg.T
    streams, bounds = _layer_streams(cfg, range(n), T)
    mk = lambda: [h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype) for _ in range(n)]  # noqa: E731
    grouped, single = mk(), mk()
    for ci in range(len(bounds)):
        if ci == 0:
            for l in range(n):
                grouped[l].prefill(*streams[l][0])
                single[l].prefill(*streams[l][0])
            continue
        outs_g = h2o.step_layers(grouped, [s[ci][0] for s in streams], [s[ci][1] for s in streams],
                                 [s[ci][2] for s in streams])
        outs_s = [single[l].step(*streams[l][ci]) for l in range(n)]
        torch.cuda.synchronize()
        for l in range(n):
            assert torch.equal(outs_g[l], outs_s[l]), f"chunk {ci} layer {l}: outputs differ"
            for x, y in zip(grouped[l].read_state() + grouped[l].read_delta(),
                            single[l].read_state() + single[l].read_delta()):
                assert torch.equal(x, y), f"chunk {ci} layer {l}: state differs"
            assert grouped[l].info()["t0"] == bounds[ci][1]
    for l in range(n):
        for x, y in zip(grouped[l].read_kv(), single[l].read_kv()):
            assert torch.equal(x, y)
    for c in grouped + single:
        c.close()


def test_step_layers_host_buffers_match_device_buffers(h2o, monkeypatch):
    """Grouped steps with host buffers (pinned, then pageable) give, bit for bit,
    what the same steps with device buffers give.  With host outputs and at least
    eight layers the step runs its layers in sub-groups, each sub-group's outputs
    copied to the host while the next one computes; the outputs are complete once
    the caller's stream has passed the step."""
    monkeypatch.setenv("H2O_ATTN_SPLIT", "1")
    cfg, n = _cfg(0, dtype=torch.bfloat16, d=128, name="tiny-bf16"), 10
    streams, bounds = _layer_streams(cfg, range(n), cfg.T)
    mk = lambda: [h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype) for _ in range(n)]  # noqa: E731
    dev, host = mk(), mk()
    for l in range(n):
        dev[l].prefill(*streams[l][0])
        host[l].prefill(*streams[l][0])
    for ci in range(1, len(bounds)):
        outs_d = h2o.step_layers(dev, [s[ci][0] for s in streams], [s[ci][1] for s in streams],
                                 [s[ci][2] for s in streams])
        pin = ci % 2 == 1
        hs = [tuple(x.cpu().pin_memory() if pin else x.cpu() for x in s[ci]) for s in streams]
        houts = [torch.empty_like(h[0]).pin_memory() if pin else torch.empty_like(h[0]) for h in hs]
        h2o.step_layers(host, [h[0] for h in hs], [h[1] for h in hs], [h[2] for h in hs], outs=houts)
        torch.cuda.synchronize()
        for l in range(n):
            assert torch.equal(outs_d[l].cpu(), houts[l]), f"chunk {ci} layer {l}: outputs differ"
            for x, y in zip(dev[l].read_state() + dev[l].read_delta(),
                            host[l].read_state() + host[l].read_delta()):
                assert torch.equal(x, y), f"chunk {ci} layer {l}: state differs"
    for c in dev + host:
        c.close()


def test_step_layers_against_the_oracle(h2o):
    """Three layers of the 28-layer workload stepped together; sampled (batch,
    KV head) caches of each layer followed by the oracle along the stream."""
    cfg = _cfg(4)
    n, T = 3, cfg.P + 3 * cfg.S
    streams, bounds = _layer_streams(cfg, [0, 13, 27], T)
    caches = [h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype) for _ in range(n)]
    heads = [(1, 2), (3, 7), (0, 5)]
    G = cfg.G
    orc = [H2OHeadOracle(cfg.M, cfg.R, G, cfg.d) for _ in range(n)]
    for ci in range(len(bounds)):
        pos_before = [o.pos.copy() for o in orc]
        if ci == 0:
            outs = [caches[l].prefill(*streams[l][0]) for l in range(n)]
        else:
            outs = h2o.step_layers(caches, [s[ci][0] for s in streams], [s[ci][1] for s in streams],
                                   [s[ci][2] for s in streams])
        torch.cuda.synchronize()
        for l in range(n):
            b, h = heads[l]
            q, k, v = (to64(x) for x in streams[l][ci])
            ref = orc[l].step(q[b, h * G:(h + 1) * G], k[b, h], v[b, h])
            where = f"layer {l} chunk {ci} (b={b}, h={h})"
            check_outputs(to64(outs[l])[b, h * G:(h + 1) * G], ref, cfg.dtype, where)
            slots, scores, pos = (x.cpu().numpy() for x in caches[l].read_state())
            annotate_boundary(orc[l], pos_before[l])
            if check_evictions(orc[l], slots[b, h], where) == "exact":
                assert np.array_equal(pos[b, h], orc[l].pos), f"{where}: slot -> position map differs"
                check_scores(scores[b, h], orc[l].score, orc[l].pos >= 0, where)
            else:
                check_tie_state(slots[b, h], pos[b, h], pos_before[l], bounds[ci][0], where)
                kc, vc = caches[l].read_kv()
                _sync_head(orc[l], kc, vc, scores, pos, b, h, bounds[ci][1])
    for c in caches:
        c.close()


def test_step_layers_argument_errors(h2o):
    from h2o_kv_cache_b200.workload import gen_batch, split_chunks
    cfg = _cfg(0, dtype=torch.bfloat16, d=128)
    Q, K, V = gen_batch(cfg, 0, device="cuda")
    ch = split_chunks(Q, K, V, cfg.bounds())
    a = h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype)
    b = h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype)
    a.prefill(*ch[0])
    with pytest.raises(h2o.H2OError) as ei:            # b is not prefilled
        h2o.step_layers([a, b], [ch[1][0]] * 2, [ch[1][1]] * 2, [ch[1][2]] * 2)
    assert ei.value.status == -3
    assert a.info()["t0"] == cfg.P                     # nothing ran
    with pytest.raises(h2o.H2OError) as ei:            # the same handle twice
        h2o.step_layers([a, a], [ch[1][0]] * 2, [ch[1][1]] * 2, [ch[1][2]] * 2)
    assert ei.value.status == -1
    a.close()
    b.close()


@pytest.mark.parametrize("case", ["tiny-fp32", "ragged-bf16", "m2k-s1k"])
def test_lr_policy(h2o, case):
    """The recency-only policy: the same attention, summed weights and scores as
    H2O, evictions by position; every step matches the oracle exactly and the
    cache holds the last M tokens."""
    cfgs = {
        "tiny-fp32": _cfg(0, name="lr-tiny"),
        "ragged-bf16": _cfg(0, name="lr-ragged", B=2, Hq=6, Hkv=2, d=128, M=300, R=17,
                            T=100 + 37 * 7 + 11, P=100, S=37, dtype=torch.bfloat16, planted=0.02),
        "m2k-s1k": _cfg(1, name="lr-m2k"),
    }
    cfg = cfgs[case]
    T = cfg.P + 4 * cfg.S if case == "m2k-s1k" else None
    heads = [(0, 2), (0, 5)] if case == "m2k-s1k" else None
    s = run_stream(h2o, cfg, heads=heads, T=T, policy="lr")
    assert s["ties"] == 0


def test_step_layers_lr_policy_against_the_oracle(h2o):
    """Grouped steps of lr caches: the same one-grid path, evictions by position."""
    cfg = _cfg(1, name="lr-m2k-layers")
    n, T = 3, cfg.P + 3 * cfg.S
    streams, bounds = _layer_streams(cfg, [0, 1, 2], T)
    caches = [h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype, policy="lr") for _ in range(n)]
    G = cfg.G
    orc = [H2OHeadOracle(cfg.M, cfg.R, G, cfg.d, "lr") for _ in range(n)]
    b, h = 0, 3
    for ci in range(len(bounds)):
        if ci == 0:
            outs = [caches[l].prefill(*streams[l][0]) for l in range(n)]
        else:
            outs = h2o.step_layers(caches, [s[ci][0] for s in streams], [s[ci][1] for s in streams],
                                   [s[ci][2] for s in streams])
        torch.cuda.synchronize()
        for l in range(n):
            q, k, v = (to64(x) for x in streams[l][ci])
            ref = orc[l].step(q[b, h * G:(h + 1) * G], k[b, h], v[b, h])
            where = f"lr layer {l} chunk {ci}"
            check_outputs(to64(outs[l])[b, h * G:(h + 1) * G], ref, cfg.dtype, where)
            slots, scores, pos = (x.cpu().numpy() for x in caches[l].read_state())
            assert np.array_equal(slots[b, h], orc[l].last_freed), f"{where}: filled slots differ"
            assert np.array_equal(pos[b, h], orc[l].pos), f"{where}: slot -> position map differs"
            check_scores(scores[b, h], orc[l].score, orc[l].pos >= 0, where)
            # the cache holds the most recent M tokens
            t = bounds[ci][1]
            assert sorted(int(x) for x in pos[b, h] if x >= 0) == list(range(max(0, t - cfg.M), t))
    for c in caches:
        c.close()
