"""The stamps tool's arithmetic (h2o_kv_cache_b200/stamps.py) on synthetic stamps:
the per-SM CTA gaps of the attention launch and the tail's phase spans (CPU only:
no GPU call)."""
import numpy as np

from h2o_kv_cache_b200 import stamps


def test_units_gaps_are_per_sm_in_start_order():
    # two SMs; SM 0 runs CTAs [1, 100) then [110, 300); SM 1 runs [5, 205) then
    # [255, 355) -- listed out of start order, plus an unstamped row
    ut = np.array([[1, 255, 355], [0, 110, 300], [0, 0, 0], [1, 5, 205], [0, 1, 100]], dtype=np.int64)
    ut[:, 1:][ut[:, 1:] > 0] += 1000          # a global timer never starts at 0
    out = stamps.summarize_units(ut)
    assert out["CTAs"] == 4
    # lives 100, 190, 200, 99 -> median 145
    assert out["CTA life, median (ns)"] == 145.0
    # gaps: SM 0 110 - 100 = 10, SM 1 255 - 205 = 50
    assert out["gap between a CTA's exit and the next CTA's entry on its SM, median (ns)"] == 30.0
    assert out["launch span (ns)"] == 355 - 1


def test_tail_phase_spans():
    # one CTA: start 100, phase boundaries at 150 / 240 / 300 / 310 / 400, one radix pass,
    # sub-stamps 7..13 inside the phases
    t = np.zeros((3, stamps.TAIL_SLOTS), dtype=np.int64)
    t[0, :6] = [100, 150, 240, 300, 310, 400]
    t[0, 6] = 1
    t[0, 7:14] = [160, 170, 200, 230, 260, 320, 250]
    out = stamps.summarize_tail(t)
    assert out["CTAs stamped"] == 1
    assert out["score accumulate and keys (phase 1)"] == 50
    assert out["selection (incl. the first barrier)"] == 90
    assert out["compaction"] == 60
    assert out["barrier before the scatter"] == 10
    assert out["scatter"] == 90
    assert out["whole kernel"] == 300
    assert out["radix passes of the selection"] == 1
    assert out["  selection: first cluster barrier"] == 10
    assert out["  selection: pass 1's merged read and decision"] == 30
    assert out["  compaction: the CTA's count published"] == 10
    assert out["  compaction: the warps' counts"] == 10
    assert out["  compaction: exchange and ordered write"] == 40
    assert out["  scatter: staged rows landed"] == 10
    assert out["  scatter: stores"] == 80
