"""Pipeline stamps of the tensor-core attention kernel (a developer tool).

    python -m h2o_kv_cache_b200.stamps [--config 4] [--layers 2] [--steps 3]

Builds the instrumented library (build.py --stamps: the attention kernel compiled
with -DH2O_STAMPS records clock64() at its hand-offs), runs a few chunk steps of
a workload on it in a child process, and prints, per 256-key pair of sweep 1 and
per 128-key tile of sweep 2, the medians over the first wave's CTAs of how long
each role waited on the others and how long the softmax took.  Needs a B200.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
import tempfile

import numpy as np

KCTAS, KSLOTS = 148, 1200
TAIL_CTAS, TAIL_SLOTS = 1024, 16
UNIT_CTAS = 16384
# slot bases, as in csrc/attn_umma.cu
ISSUE_K, K_FULL, S_EMPTY, PAIR_ISSUED, S_FULL, PAIR_END = 0, 64, 128, 256, 320, 448
ST_START, ST_READY, OT_READY, ST_FULL, P_EMPTY, P_FULL = 512, 608, 704, 800, 896, 992
START, SWEEP1_END, SWEEP2_END = 1100, 1101, 1102


def _child(cfg_id, layers, steps, out_path):
    import ctypes
    import dataclasses

    import torch

    import h2o_kv_cache_b200 as h2o
    from h2o_kv_cache_b200.workload import CONFIGS, gen_batch, split_chunks
    cfg = dataclasses.replace(CONFIGS[cfg_id], layers=layers)
    T = cfg.P + (steps + 1) * cfg.S
    bounds = [(a, b) for a, b in cfg.bounds() if a < T]
    caches, chunks = [], []
    for layer in range(cfg.layers):
        Q, K, V = gen_batch(cfg, layer, device="cuda", T=T)
        ch = split_chunks(Q, K, V, bounds)
        c = h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype)
        c.prefill(*ch[0])
        caches.append(c)
        chunks.append(ch)
    for i in range(1, min(steps + 1, len(bounds))):
        if len(caches) > 1:
            h2o.step_layers(caches, [c[i][0] for c in chunks], [c[i][1] for c in chunks],
                            [c[i][2] for c in chunks])
        else:
            caches[0].step(*chunks[0][i])
    torch.cuda.synchronize()
    buf = (ctypes.c_ulonglong * (KCTAS * KSLOTS))()
    tbuf = (ctypes.c_ulonglong * (TAIL_CTAS * TAIL_SLOTS))()
    ubuf = (ctypes.c_ulonglong * (UNIT_CTAS * 3))()
    if (h2o.lib.h2o_stamps_read(buf) != 0 or h2o.lib.h2o_tail_stamps_read(tbuf) != 0
            or h2o.lib.h2o_unit_stamps_read(ubuf) != 0):
        raise RuntimeError("reading the stamps failed")
    tail = np.frombuffer(tbuf, dtype=np.uint64).reshape(TAIL_CTAS, TAIL_SLOTS).astype(np.int64)
    # the launch floor of the tail's shape: an empty kernel with the same grid
    # and cluster size (90 KB of shared memory), timed between CUDA events right
    # after a busy kernel, as the step's tail launch is
    n_cta = int((tail[:, 0] > 0).sum())
    n_caches = cfg.B * cfg.Hkv * cfg.layers
    floor_us = float("nan")
    if 0 < n_cta < TAIL_CTAS and n_cta % n_caches == 0 and n_cta // n_caches <= 16:
        st = torch.cuda.current_stream()
        times = []
        for _ in range(25):
            torch.cuda._sleep(200000)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            if h2o.lib.h2o_tail_empty_launch(n_cta // n_caches, n_cta, 90 * 1024, 1, st.cuda_stream) != 0:
                raise RuntimeError("empty launch failed")
            b.record(st)
            b.synchronize()
            times.append(a.elapsed_time(b) * 1e3)
        floor_us = float(np.median(times[5:]))
    np.savez(out_path, attn=np.frombuffer(buf, dtype=np.uint64).reshape(KCTAS, KSLOTS).astype(np.int64),
             tail=tail, unit=np.frombuffer(ubuf, dtype=np.uint64).reshape(UNIT_CTAS, 3).astype(np.int64),
             floor_us=np.array(floor_us))


def summarize_tail(tt):
    """Median (over CTAs) of each phase of the tail kernel, in SM clock cycles."""
    ok = (tt[:, 0] > 0) & (tt[:, 5] > tt[:, 0])
    if not ok.any():
        return {}
    t = tt[ok]
    names = ["score accumulate and keys (phase 1)", "selection (incl. the first barrier)",
             "compaction", "barrier before the scatter", "scatter", "whole kernel"]
    spans = [t[:, 1] - t[:, 0], t[:, 2] - t[:, 1], t[:, 3] - t[:, 2], t[:, 4] - t[:, 3],
             t[:, 5] - t[:, 4], t[:, 5] - t[:, 0]]
    out = {nm: float(np.median(x)) for nm, x in zip(names, spans)}
    out["radix passes of the selection"] = float(np.median(t[:, 6]))
    if (t[:, 10] > 0).all():
        out["  selection: first cluster barrier"] = float(np.median(t[:, 7] - t[:, 1]))
        out["  selection: pass 1's local histogram"] = float(np.median(t[:, 8] - t[:, 7]))
        out["  selection: pass 1's remote adds and barrier"] = float(np.median(t[:, 9] - t[:, 8]))
        out["  selection: pass 1's merged read and decision"] = float(np.median(t[:, 10] - t[:, 9]))
    if (t[:, 11] > 0).all():
        if (t[:, 13] > 0).all():
            out["  compaction: the CTA's count published"] = float(np.median(t[:, 13] - t[:, 2]))
            out["  compaction: the warps' counts"] = float(np.median(t[:, 11] - t[:, 13]))
        else:
            out["  compaction: counts"] = float(np.median(t[:, 11] - t[:, 2]))
        out["  compaction: exchange and ordered write"] = float(np.median(t[:, 3] - t[:, 11]))
    if (t[:, 12] > 0).all():
        out["  scatter: staged rows landed"] = float(np.median(t[:, 12] - t[:, 4]))
        out["  scatter: stores"] = float(np.median(t[:, 5] - t[:, 12]))
    out["CTAs stamped"] = float(ok.sum())
    return out


def summarize_units(ut):
    """The attention launch's CTAs per SM in start order: each CTA's life and
    the gap before the next CTA on its SM, global-timer nanoseconds."""
    ok = (ut[:, 1] > 0) & (ut[:, 2] > ut[:, 1])
    if ok.sum() < 2:
        return {}
    sm, t0, t1 = ut[ok, 0], ut[ok, 1], ut[ok, 2]
    gaps, lives = [], t1 - t0
    for s_ in np.unique(sm):
        idx = np.nonzero(sm == s_)[0]
        order = idx[np.argsort(t0[idx])]
        gaps.extend((t0[order[1:]] - t1[order[:-1]]).tolist())
    out = {"CTAs": float(ok.sum()), "CTA life, median (ns)": float(np.median(lives)),
           "launch span (ns)": float(t1.max() - t0.min())}
    if gaps:
        out["gap between a CTA's exit and the next CTA's entry on its SM, median (ns)"] = float(np.median(gaps))
        out["  p90 (ns)"] = float(np.percentile(gaps, 90))
    return out


def summarize(st):
    """Median (over CTAs) of per-CTA mean waits, in SM clock cycles."""
    out = {}
    s1 = []
    for c in range(st.shape[0]):
        end = st[c, PAIR_END:PAIR_END + 64]
        n = int((end > 0).sum())
        if n < 4:
            continue
        u = np.arange(2, n - 1)
        s1.append([(end[u] - end[u - 1]).mean(),
                   (st[c, S_FULL + u] - end[u - 1]).mean(),
                   (st[c, S_FULL + 64 + u] - st[c, S_FULL + u]).mean(),
                   (end[u] - st[c, S_FULL + 64 + u]).mean(),
                   (st[c, K_FULL + u] - st[c, PAIR_ISSUED + u - 1]).mean(),
                   (st[c, S_EMPTY + u] - st[c, K_FULL + u]).mean(),
                   (st[c, S_FULL + u] - st[c, S_EMPTY + u]).mean()])
    names1 = ["period per 256-key pair", "softmax waits for head A's S", "head A (softmax, then waits for B's S)",
              "head B softmax", "MMA warp waits for the K tile", "MMA warp waits for head A's S buffer",
              "head A's S: MMA issue to the softmax's S full"]
    if s1:
        out["sweep 1"] = dict(zip(names1, np.median(np.array(s1), axis=0)))
    s2 = []
    for c in range(st.shape[0]):
        pf = st[c, P_FULL:P_FULL + 96]
        n = int((pf > 0).sum())
        if n < 6:
            continue
        j = np.arange(2, n - 1)
        s2.append([(pf[j] - pf[j - 1]).mean(),
                   (st[c, ST_FULL + j] - pf[j - 1]).mean(),
                   (st[c, P_EMPTY + j] - st[c, ST_FULL + j]).mean(),
                   (pf[j] - st[c, P_EMPTY + j]).mean(),
                   (st[c, ST_READY + j] - st[c, ST_START + j]).mean(),
                   (st[c, OT_READY + j - 1] - st[c, ST_READY + j]).mean(),
                   (st[c, ST_FULL + j] - st[c, ST_READY + j]).mean()])
    names2 = ["period per 128-key tile", "softmax waits for S^T", "exponentials (and wait for the P^T buffer)",
              "P^T stores", "MMA warp waits before S^T", "MMA warp waits before O^T",
              "S^T: MMA issue to the softmax's S^T full"]
    if s2:
        out["sweep 2"] = dict(zip(names2, np.median(np.array(s2), axis=0)))
    ok = st[:, START] > 0
    out["unit"] = {"start to end of sweep 1": float(np.median(st[ok, SWEEP1_END] - st[ok, START])),
                   "start to end of sweep 2": float(np.median(st[ok, SWEEP2_END] - st[ok, START]))}
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", type=int, default=4)
    ap.add_argument("--layers", type=int, default=2)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--save", default=None, help="also keep the raw stamps (.npz) here")
    ap.add_argument("--child", default=None, help=argparse.SUPPRESS)
    args = ap.parse_args()
    if args.child:
        _child(args.config, args.layers, args.steps, args.child)
        return
    here = os.path.dirname(os.path.abspath(__file__))
    sys.path.insert(0, here)
    import build as B
    lib = B.build(stamps=True)
    out = os.path.join(tempfile.mkdtemp(), "stamps.npz")
    env = dict(os.environ, H2O_LIBRARY=lib)
    subprocess.run([sys.executable, "-m", "h2o_kv_cache_b200.stamps", "--config", str(args.config),
                    "--layers", str(args.layers), "--steps", str(args.steps), "--child", out],
                   check=True, env=env, cwd=os.path.dirname(here))
    data = np.load(out)
    if args.save:
        shutil.copyfile(out, args.save)
    res = summarize(data["attn"])
    res["tail (one launch: the last step's)"] = summarize_tail(data["tail"])
    res["tensor-core attention CTAs (its last launch)"] = summarize_units(data["unit"])
    if "floor_us" in data and np.isfinite(data["floor_us"]):
        res["tail launch floor (an empty kernel of its shape, CUDA events)"] = {
            "nanoseconds": float(data["floor_us"]) * 1e3}
    print(f"workload config {args.config}, {args.layers} layer(s), last of {args.steps} steps; "
          "medians over the first wave's CTAs, SM clock cycles")
    for part, vals in res.items():
        print(part)
        for k, v in vals.items():
            print(f"  {k:48s} {v:10.0f}")


if __name__ == "__main__":
    main()
