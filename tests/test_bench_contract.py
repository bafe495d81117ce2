"""bench.py's arithmetic and its reference arm, on the CPU.

The roofline figures of the bench line rest on two counts: algorithmic FLOPs
per attention launch (4 d per (query-head row, visible key) pair: QK^T and PV,
the recompute of the second sweep not credited) and algorithmic bytes of score
accumulate + select + scatter.  The FLOP counts are checked against the
per-step figures derived independently for the measurement table of the
workloads (42.96, 283.5, 1134 and 584 GFLOP for a full cache and one chunk),
and the reference arm is run once to check its JSON line.
"""
import importlib.util
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("cid,gflop", [(1, 42.96), (2, 283.5), (3, 1134.0), (4, 584.0)])
def test_flops_per_step_match_the_measurement_table(cid, gflop):
    from h2o_kv_cache_b200.workload import CONFIGS
    b = _bench()
    cfg = CONFIGS[cid]
    flops = 4 * cfg.d * b.attn_pairs(cfg, cfg.S, cfg.M)     # full cache, one chunk, one layer
    assert abs(flops / 1e9 - gflop) / gflop < 1e-3, flops / 1e9


def test_pairs_count_visible_keys():
    # a brute count of (row, visible key) pairs on a small case
    from h2o_kv_cache_b200.workload import Config
    import torch
    b = _bench()
    cfg = Config(9, "t", 2, 6, 3, 16, 40, 4, 100, 40, 7, torch.float32, 0.0)
    S, nv = 7, 40
    brute = sum(nv + (i + 1) for _ in range(cfg.B * cfg.Hq) for i in range(S))
    assert b.attn_pairs(cfg, S, nv) == brute


def test_select_scatter_bytes():
    from h2o_kv_cache_b200.workload import CONFIGS
    b = _bench()
    cfg = CONFIGS[1]
    # scores and positions (4 B each) read and written for every slot, and the
    # chunk's K and V rows (bf16) read and written, per (batch, KV head)
    expect = cfg.B * cfg.Hkv * (cfg.M * 8 * 2 + cfg.S * cfg.d * 2 * 2 * 2)
    assert b.select_scatter_bytes(cfg, cfg.S) == expect == 8650752


def test_reference_arm_prints_one_json_line():
    # the reference arm on the default workload (28 layers, B=4): one oracle step per timed step
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["metric"] == "H2O chunk-step query-tokens/s" and d["unit"] == "query-tokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["os_cpu_count"] == os.cpu_count()
    # the same config object as the GPU arm prints, and the time it measured per step
    b = _bench()
    from h2o_kv_cache_b200.workload import CONFIGS
    assert d["config"] == b.config_dict(CONFIGS[4], 1)
    ex = d["extrapolation"]
    assert abs(ex["ms_per_workload_step"] - d["ms_per_step"] * ex["caches_per_workload_step"]) < 1e-6 * ex["ms_per_workload_step"]
    assert ex["caches_per_workload_step"] == 4 * 8 * 28


def test_reference_arm_maps_no_product_library():
    # the oracle arm loads the input generator from its file, not through the
    # package (whose import loads libh2o.so)
    code = ("import sys, runpy; sys.argv = ['bench.py', '--impl', 'reference', '--steps', '1', "
            "'--warmup', '3', '--config', '0']; runpy.run_path('bench.py', run_name='__main__'); "
            "maps = open('/proc/self/maps').read(); print('MAPPED' if 'libh2o' in maps else 'CLEAN')")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip().splitlines()[-1] == "CLEAN"


def test_roofline_objects_arithmetic():
    # achieved = algorithmic FLOPs (bytes) per launch / the launch's time; the
    # 28-layer workload is read against the sustained peak, one layer against
    # the burst peak
    from h2o_kv_cache_b200.workload import CONFIGS
    b = _bench()
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "source": "measured"}
    res = {"flops": 700e9, "attn_ms": 1.0, "sel_ms": 0.01}
    for cid, peak in ((4, 1400.0), (1, 1600.0)):
        cfg = CONFIGS[cid]
        att, sel = b.roofline_objects(cfg, res, peaks)
        assert att["achieved"] == pytest.approx(700.0)
        assert att["peak"] == peak and att["frac"] == pytest.approx(700.0 / peak)
        assert att["frac_of_burst_peak"] == pytest.approx(700.0 / 1600.0)
        gbs = b.select_scatter_bytes(cfg, cfg.S) / 1e-5 / 1e9
        assert sel["achieved"] == pytest.approx(gbs) and sel["frac"] == pytest.approx(gbs / 6000.0)


def test_traffic_is_null_once_the_sources_change(tmp_path, monkeypatch):
    # a DRAM-bytes entry counts only while the attention path's sources hash to
    # the value it was captured on
    from h2o_kv_cache_b200.workload import CONFIGS
    b = _bench()
    csrc = tmp_path / "h2o_kv_cache_b200" / "csrc"
    csrc.mkdir(parents=True)
    for n in b.KERNEL_SOURCES["fused"]:
        (csrc / n).write_text("// " + n + "\n")
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    cfg = CONFIGS[4]
    (tmp_path / "profiles").mkdir()
    entry = {cfg.name: {"path": "fused", "sources_sha": b.sources_sha(b.KERNEL_SOURCES["fused"]),
                        "dram_bytes_per_launch": 123.0}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(entry))
    assert b.traffic_for(cfg) == 123.0
    (csrc / b.KERNEL_SOURCES["fused"][0]).write_text("// changed\n")
    assert b.traffic_for(cfg) is None


def test_committed_traffic_entries_name_known_paths():
    b = _bench()
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        entries = json.load(f)
    for name, ent in entries.items():
        assert ent["path"] in b.KERNEL_SOURCES, name
        assert ent["dram_bytes_per_launch"] > 0, name
        assert os.path.exists(os.path.join(ROOT, ent["source"])), name
