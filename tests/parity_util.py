"""GPU-vs-oracle comparison for the H2O chunk step (used by the -m gpu tests).

Tolerances (written here, used by every parity test):
  outputs  float32: |gpu - ref| <= 1e-4 * max_c |ref[..., c]| (each output row's
           largest component), elementwise
           bfloat16: |gpu - ref| <= 2e-2 absolute, and per (chunk, batch, KV head)
           ||gpu - ref|| / ||ref|| <= 1e-2 (outputs of near-uniform attention over
           thousands of keys are ~1e-2 in size, so the absolute bound alone would
           pass a PV product that dropped a whole V tile; bf16 rounding of P and
           of the output gives a relative norm error of a few 1e-3)
  scores   |gpu - ref| <= 1e-3 * |ref|
  evicted slots and slot -> position maps: bit-exact where the oracle's rank gap
  at the eviction boundary exceeds 1e-3; otherwise every slot in the symmetric
  difference must score within 1e-3 (relative) of the boundary score, and the
  oracle is then re-synchronised to the GPU's state before the next chunk.
"""
from __future__ import annotations

import numpy as np
import torch

OUT_RTOL_F32 = 1e-4
OUT_ATOL_BF16 = 2e-2
OUT_RELNORM_BF16 = 1e-2
SCORE_RTOL = 1e-3
GAP_TOL = 1e-3


def to64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def check_outputs(gpu, ref, dtype, where=""):
    """gpu, ref: float64 arrays of the same shape."""
    err = np.abs(gpu - ref)
    if dtype == torch.float32:
        # relative to each output row's magnitude (its largest component): an
        # elementwise relative bound is undefined where a component crosses zero
        row = np.abs(ref).max(axis=-1, keepdims=True)
        bound = OUT_RTOL_F32 * np.maximum(row, 1e-30)
        bad = err > bound
        assert not bad.any(), (f"{where}: {int(bad.sum())} fp32 outputs out of tolerance, "
                               f"max err {err.max():.3e}")
    rel = float(np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-30))
    if dtype != torch.float32:
        assert err.max() <= OUT_ATOL_BF16, f"{where}: bf16 output max err {err.max():.3e}"
        assert rel <= OUT_RELNORM_BF16, f"{where}: bf16 output relative norm error {rel:.3e}"
    return {"max_abs": float(err.max()) if err.size else 0.0, "rel_norm": rel}


def check_scores(gpu, ref, valid, where=""):
    g, r = gpu[valid], ref[valid]
    err = np.abs(g - r)
    bad = err > SCORE_RTOL * np.abs(r)
    assert not bad.any(), (f"{where}: {int(bad.sum())} scores out of tolerance, worst rel "
                           f"{float((err / np.maximum(np.abs(r), 1e-30)).max()):.3e}")
    return float((err / np.maximum(np.abs(r), 1e-30)).max()) if g.size else 0.0


def rank_gap(pre_scores, pos, eligible, need):
    """Relative gap at the eviction boundary among the eligible slots, by (score, pos)."""
    idx = np.nonzero(eligible)[0]
    if need == 0 or need >= idx.size:
        return np.inf
    order = np.lexsort((pos[idx], pre_scores[idx]))
    s = pre_scores[idx][order]
    lo, hi = s[need - 1], s[need]
    return (hi - lo) / max(abs(lo), 1e-30)


def check_evictions(head, gpu_freed, where=""):
    """head: oracle head after its step; gpu_freed: the GPU's filled slots for that
    head.  Returns 'exact', or 'ties' when the sets differ only within a near-tie
    (the caller then re-synchronises the oracle)."""
    need = head.last_need
    ref = np.asarray(head.last_freed)
    got = np.asarray(gpu_freed)
    assert got.shape == ref.shape, f"{where}: freed length {got.shape} vs {ref.shape}"
    if np.array_equal(got, ref):
        return "exact"
    pre, pos_before = head.last_pre_scores, None
    gap = head.last_gap
    ref_ev, got_ev = set(ref[:need].tolist()), set(got[:need].tolist())
    assert np.array_equal(got[need:], ref[need:]), f"{where}: empty-slot fill order differs"
    assert gap <= GAP_TOL, (f"{where}: eviction sets differ with rank gap {gap:.3e} > {GAP_TOL} "
                            f"(gpu-only {sorted(got_ev - ref_ev)[:8]}, oracle-only "
                            f"{sorted(ref_ev - got_ev)[:8]})")
    boundary = head.last_boundary
    for s in ref_ev ^ got_ev:
        assert head.last_eligible[s], f"{where}: GPU evicted an ineligible slot {s}"
        assert abs(pre[s] - boundary) <= GAP_TOL * abs(boundary), (
            f"{where}: slot {s} score {pre[s]} is not within {GAP_TOL} of the boundary {boundary}")
    assert np.all(np.diff(got) > 0), f"{where}: filled slots not strictly ascending (duplicates?)"
    return "ties"


def check_tie_state(gpu_freed, gpu_pos, pos_before, t0, where=""):
    """Validity of a step whose eviction set the oracle does not fix (a near-tie):
    the filled slots are unique and ascending, chunk token t0 + i sits in the
    i-th filled slot, each new token appears exactly once, and every slot that was
    not filled kept the position it held before the step."""
    freed = np.asarray(gpu_freed)
    pos = np.asarray(gpu_pos)
    before = np.asarray(pos_before)
    S = freed.size
    assert np.all(np.diff(freed) > 0), f"{where}: filled slots not strictly ascending"
    assert freed.min() >= 0 and freed.max() < pos.size, f"{where}: filled slot out of range"
    assert np.array_equal(pos[freed], t0 + np.arange(S)), f"{where}: slot -> new token map wrong"
    new = np.sort(pos[pos >= t0])
    assert np.array_equal(new, t0 + np.arange(S)), f"{where}: new tokens not each cached once"
    kept = np.ones(pos.size, bool)
    kept[freed] = False
    assert np.array_equal(pos[kept], before[kept]), f"{where}: a slot not filled changed position"


def annotate_boundary(head, pos_before):
    """Record the oracle's rank gap and boundary score for the last step."""
    need = head.last_need
    elig = head.last_eligible
    head.last_gap = rank_gap(head.last_pre_scores, pos_before, elig, need)
    if need > 0:
        idx = np.nonzero(elig)[0]
        order = np.lexsort((pos_before[idx], head.last_pre_scores[idx]))
        head.last_boundary = head.last_pre_scores[idx][order][need - 1]
    else:
        head.last_boundary = 0.0
