"""Position-indexed brute force of chunked H2O attention, for tiny inputs.

TEST INFRASTRUCTURE ONLY (same import rule as ``oracle/h2o_oracle.py``).

A second, deliberately different formulation of the method of "Learning how to
Forget: Fine-tuning for Long-Context Sparse Attention" (Abstract; §1 ¶1 fixed-size
cache with eviction; FAQ answer 3 summed attention weights; Figure 1(a) chunks).
It keeps no slots: the cache is a boolean mask over the whole stream's positions
and each score is a per-position value.  Every query row is an explicit dense
masked softmax over *all* stream positions, computed one row at a time with
Python-level loops over the mask.  It shares no code with the slot oracle, so
the slot oracle's bookkeeping (slot reuse, score carry-over, scatter) can be
checked against it.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = ["brute_stream"]


def brute_stream(Q, K, V, M, R, prefill, chunk):
    """Run a whole stream.

    Q [Hq, T, d], K, V [Hkv, T, d] (one batch element), prefill length P, then
    chunks of `chunk` tokens (the last may be shorter).
    Returns dict with
      outs    [Hq, T, d]      every token's attention output
      cached  list per chunk of the sorted cached positions after the chunk, per KV head
      scores  list per chunk of {pos: score} after the chunk, per KV head
    """
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    Hq, T, d = Q.shape
    Hkv = K.shape[0]
    G = Hq // Hkv
    scale = 1.0 / math.sqrt(d)
    outs = np.zeros((Hq, T, d))
    in_cache = np.zeros((Hkv, T), dtype=bool)
    score = np.zeros((Hkv, T))
    cached_hist, score_hist = [], []
    bounds = [(0, prefill)]
    t = prefill
    while t < T:
        bounds.append((t, min(T, t + chunk)))
        t += chunk
    for (t0, t1) in bounds:
        mass = np.zeros((Hkv, T))
        for hq in range(Hq):
            h = hq // G
            for i in range(t0, t1):
                visible = in_cache[h].copy()
                visible[t0:i + 1] = True
                idx = [p for p in range(T) if visible[p]]
                logits = np.array([scale * float(Q[hq, i] @ K[h, p]) for p in idx])
                w = np.exp(logits - logits.max())
                w = w / w.sum()
                o = np.zeros(d)
                for wi, p in zip(w, idx):
                    o += wi * V[h, p]
                    mass[h, p] += wi
                outs[hq, i] = o
        S = t1 - t0
        for h in range(Hkv):
            score[h, in_cache[h]] += mass[h, in_cache[h]]
            n_in = int(in_cache[h].sum())
            need = max(0, n_in + S - M)
            cand = [p for p in range(T) if in_cache[h, p] and p < t0 - R]
            cand.sort(key=lambda p: (score[h, p], p))
            if need > len(cand):
                raise ValueError("not enough evictable positions")
            for p in cand[:need]:
                in_cache[h, p] = False
                score[h, p] = 0.0
            for p in range(t0, t1):
                in_cache[h, p] = True
                score[h, p] = mass[h, p]
        cached_hist.append([sorted(np.nonzero(in_cache[h])[0].tolist()) for h in range(Hkv)])
        score_hist.append([{p: score[h, p] for p in np.nonzero(in_cache[h])[0].tolist()}
                           for h in range(Hkv)])
    return {"outs": outs, "cached": cached_hist, "scores": score_hist}
