"""Benchmark of the H2O chunk step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

One step = one chunk of S query tokens through the whole path (attention with
summed weights, score accumulate, select, scatter) on every layer's caches.  The
default workload is the largest single-GPU one: B=4 sequences, 28 independent
layer caches (Hq=32, Hkv=8, d=128, M=8192, R=512, bf16), chunks of S=1024; a step
runs the chunk through all 28 layers.  The 16k-slot / 1k-chunk and 32k-slot /
2k-chunk single-layer workloads are measured in the same run and reported under
"other_workloads" (their attention and select/scatter roofline figures).
Inputs are resident in HBM before timing; L2 is flushed (a 256 MiB write)
between steps, outside the per-step CUDA events.  At N > 1 GPUs every rank runs
an independent replica on its own seeded stream (the path has no cross-GPU
exchange); the time is the max over ranks.

Prints ONE JSON line (rank 0).  `--impl reference` times the float64 CPU oracle
instead, on a bounded sample of the same workload (rank 0 only); it loads no
part of the CUDA library.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "H2O chunk-step query-tokens/s"
PROF_EVERY = 8     # timed steps per step with per-kernel events
UNIT = "query-tokens/s"
L2_FLUSH_BYTES = 256 << 20


def workload_module():
    """The seeded input generator, loaded from its file: importing it through the
    package would load libh2o.so, which the reference arm must not map."""
    import importlib.util
    name = "h2o_bench_workload"
    if name in sys.modules:
        return sys.modules[name]
    spec = importlib.util.spec_from_file_location(
        name, os.path.join(ROOT, "h2o_kv_cache_b200", "workload.py"))
    mod = importlib.util.module_from_spec(spec)
    sys.modules[name] = mod
    spec.loader.exec_module(mod)
    return mod


def config_dict(cfg, world):
    """The `config` object of the JSON line; both arms print the same one."""
    return {"workload": f"{cfg.name}: {cfg.describe()}", "global_batch": cfg.B * world,
            "seq_len": cfg.S, "layers": cfg.layers,
            "parallelism": f"replicas x{world}" if world > 1 else "single",
            "l2": "flushed between steps (256 MiB write outside the per-step events)"}


def host_cores():
    return {"blas_threads": blas_threads(), "os_cpu_count": os.cpu_count()}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def attn_pairs(cfg, S, n_valid):
    """(query-head row, visible key) pairs of one step: B*Hq*(S*n_valid + S(S+1)/2)."""
    return cfg.B * cfg.Hq * (S * n_valid + S * (S + 1) // 2)


def select_scatter_bytes(cfg, S):
    """Algorithmic bytes of score accumulate + select + scatter for one step:
    scores and positions read and written once, the chunk's K/V rows read and
    written once, the new scores written."""
    BH = cfg.B * cfg.Hkv
    es = 2 if cfg.dtype == torch.bfloat16 else 4
    state = BH * cfg.M * (4 + 4) * 2
    rows = BH * S * cfg.d * es * 2 * 2
    return state + rows


CLOCK_REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
                 0x40: "hw_thermal_slowdown"}   # NVML clock-event reason bits


def clock_poller(index, period_s=0.0005):
    """Child process of ClockSampler: polls NVML every period_s until its standard
    input closes, then prints one JSON line of (SM MHz, reason bits) samples.  A
    process of its own, so that the bench's Python thread never delays it."""
    import threading
    import pynvml as nv
    nv.nvmlInit()
    hdl = nv.nvmlDeviceGetHandleByIndex(index)
    smax = nv.nvmlDeviceGetMaxClockInfo(hdl, nv.NVML_CLOCK_SM)
    done = threading.Event()
    threading.Thread(target=lambda: (sys.stdin.read(), done.set()), daemon=True).start()
    print("ready", flush=True)
    samples = []
    while not done.is_set():
        try:
            samples.append((nv.nvmlDeviceGetClockInfo(hdl, nv.NVML_CLOCK_SM),
                            int(nv.nvmlDeviceGetCurrentClocksThrottleReasons(hdl))))
        except Exception:  # noqa: BLE001 - a failed sample is skipped
            pass
        time.sleep(period_s)
    print(json.dumps({"max": smax, "samples": samples}), flush=True)


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled during a region.

    A child process polls NVML every 0.5 ms from __enter__ to __exit__ (the timed
    steps run for tens of milliseconds, far shorter than nvidia-smi's sampling
    period); without NVML, nvidia-smi samples every 100 ms instead."""

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.nvml = None
        self.result = None
        self.source = None
        self.path = os.path.join(tempfile.gettempdir(), f"h2o_bench_clocks_gpu{index}.csv")

    def __enter__(self):
        try:
            import pynvml  # noqa: F401 - only probes that NVML is importable
            self.nvml = subprocess.Popen(
                [sys.executable, os.path.abspath(__file__), "--clock-poller", str(self.index)],
                stdin=subprocess.PIPE, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            if self.nvml.stdout.readline().strip() == "ready":
                self.source = "nvml, 0.5 ms"
                return self
            self.nvml.kill()
            self.nvml.wait()
        except (ImportError, OSError):
            pass
        self.nvml = None
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index),
                 "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
            self.source = "nvidia-smi, 100 ms"
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.nvml is not None:
            try:
                out, _ = self.nvml.communicate(timeout=10)
                self.result = json.loads(out.strip().splitlines()[-1])
            except (subprocess.TimeoutExpired, ValueError, IndexError):
                self.nvml.kill()
                self.nvml.wait()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.nvml is not None:
            if self.result is None:
                return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock poller failed"]}
            smp = self.result["samples"]
            sm = [float(m) for m, _ in smp]
            reasons = sorted({n for _, b in smp for bit, n in CLOCK_REASONS.items() if b & bit})
            return {"sm_mhz": statistics.median(sm) if sm else None,
                    "sm_max_mhz": float(self.result["max"]), "reasons": reasons,
                    "samples": len(sm), "source": self.source}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    sm.append(float(parts[0]))
                    smax = float(parts[1])
                except ValueError:
                    continue
                for n, v in zip(names, parts[4:8]):
                    if v.lower() == "active":
                        reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm), "source": self.source}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()


def max_over_ranks(x, world):
    from h2o_kv_cache_b200.replicas import max_over_ranks as _max
    return _max(x, world, device="cuda")


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_sample(cfg, chunks_host, budget_s, max_head_chunks=None):
    """Times the float64 oracle on (batch 0, KV head h) caches, chunk after chunk,
    until about budget_s seconds of step work are done.  Returns
    (tokens/s extrapolated to the whole step, description, head-chunks timed)."""
    from oracle import H2OHeadOracle
    G = cfg.G
    done, elapsed, heads_used = 0, 0.0, 0
    for h in range(cfg.Hkv):
        st = H2OHeadOracle(cfg.M, cfg.R, G, cfg.d)
        q0, k0, v0 = chunks_host[0]
        st.step(q0[0, h * G:(h + 1) * G], k0[0, h], v0[0, h])           # prefill, untimed
        heads_used += 1
        for (q, k, v) in chunks_host[1:]:
            t = time.perf_counter()
            st.step(q[0, h * G:(h + 1) * G], k[0, h], v[0, h])
            elapsed += time.perf_counter() - t
            done += 1
            if elapsed >= budget_s or (max_head_chunks and done >= max_head_chunks):
                break
        if elapsed >= budget_s or (max_head_chunks and done >= max_head_chunks):
            break
    scale = cfg.B * cfg.Hkv * cfg.layers
    per_step = elapsed / done * scale
    rate = cfg.B * cfg.S / per_step
    desc = (f"float64 oracle, {done} (KV head, chunk) steps of batch 0 over {heads_used} head(s) "
            f"in {elapsed:.1f} s, extrapolated x{scale} (batch, layer, KV head) caches per step")
    return rate, desc, done, elapsed


def run_reference(args, cfg):
    """--impl reference: the oracle as it stands.  Each timed step is one
    (batch 0, layer 0, KV head 0) cache taking one chunk; ms_per_step is that
    measured time, and `value` extrapolates it to the whole workload step (all
    batch x layer x KV head caches, which the oracle would run one after the
    other).  Only rank 0 works; no part of the CUDA library is loaded."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    wl = workload_module()
    from oracle import H2OHeadOracle
    n_needed = args.warmup + args.steps
    n_ch = max(1, min(n_needed, cfg.n_chunks))
    T = min(cfg.T, cfg.P + cfg.S * n_ch)
    Q, K, V = wl.gen_sequence(cfg, 0, 0, device="cpu", T=T)
    G = cfg.G
    q_all, k_all, v_all = (x[:G] if x is Q else x[:1] for x in (Q, K, V))
    bounds = [(a, b) for a, b in cfg.bounds() if a < T]
    ch = [(q_all[:, a:b].double().numpy(), k_all[0, a:b].double().numpy(), v_all[0, a:b].double().numpy())
          for a, b in bounds]
    st = H2OHeadOracle(cfg.M, cfg.R, G, cfg.d)
    st.step(*ch[0])                                                      # prefill, untimed
    times = []
    for i in range(n_needed):
        q, k, v = ch[1 + i % (len(ch) - 1)]
        t = time.perf_counter()
        st.step(q, k, v)
        dt = time.perf_counter() - t
        if i >= args.warmup:
            times.append(dt)
    per_head_s = statistics.mean(times)
    caches = cfg.B * cfg.Hkv * cfg.layers
    value = cfg.B * cfg.S / (per_head_s * caches)
    cores = host_cores()
    sample = (f"each timed step: the float64 oracle on one (batch 0, layer 0, KV head 0) cache taking "
              f"one chunk; value extrapolates x{caches} (batch, layer, KV head) caches to a whole step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_head_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(cfg, world),
            "extrapolation": {"caches_per_workload_step": caches,
                              "ms_per_workload_step": per_head_s * caches * 1e3,
                              "ms_per_step_is": "one (batch, layer, KV head) cache, measured"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores["blas_threads"],
                             "os_cpu_count": cores["os_cpu_count"], "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def traffic_for(cfg):
    """DRAM bytes per attention launch from one ncu capture, while the sources
    it was taken on are unchanged; None otherwise."""
    tfile = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(tfile):
        return None
    try:
        with open(tfile) as f:
            ent = json.load(f).get(cfg.name)
        if ent and ent.get("sources_sha") == sources_sha(KERNEL_SOURCES[ent["path"]]):
            return ent["dram_bytes_per_launch"]
    except (OSError, ValueError, KeyError):
        pass
    return None


def measure(args, cfg, world, rank, local, steps, with_e2e):
    """Times `steps` steps of workload cfg on this rank's GPU; returns a dict of
    figures (device-timed value, per-kernel times, roofline, e2e)."""
    import h2o_kv_cache_b200 as h2o
    wl = workload_module()
    from h2o_kv_cache_b200.replicas import aggregate_throughput, replica_stream_layer
    dev = torch.device("cuda", local if world > 1 else 0)
    n_needed = args.warmup + (2 if with_e2e else 1) * steps + 1
    n_chunks = min(cfg.n_chunks, n_needed)
    T = cfg.P + cfg.S * n_chunks
    bounds = [(a, b) for a, b in cfg.bounds() if a < T]
    layers = []                                    # per layer: (cache, chunks)
    for layer in range(cfg.layers):
        # each replica (rank) has its own seeded streams
        Q, K, V = wl.gen_batch(cfg, replica_stream_layer(rank, layer), device=dev, T=T)
        chunks = wl.split_chunks(Q, K, V, bounds)
        del Q, K, V
        cache = h2o.H2OCache(cfg.M, cfg.R, cfg.Hq, cfg.Hkv, cfg.d, cfg.dtype, device=dev)
        cache.prefill(*chunks[0], want_out=False)
        layers.append((cache, chunks))
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    outs = [torch.empty_like(layers[0][1][1][0]) for _ in layers]
    n_avail = len(bounds) - 1
    ci = 0

    grouped = len(layers) > 1
    caches = [c for c, _ in layers]

    def step_all(out_bufs, host=None):
        """One step: the next chunk through every layer's cache (several layers:
        one h2o_step_layers call, i.e. one attention and one tail launch)."""
        nonlocal ci
        cs = [host[li] if host is not None else chunks[1 + ci % n_avail]
              for li, (_, chunks) in enumerate(layers)]
        if grouped:
            h2o.step_layers(caches, [c[0] for c in cs], [c[1] for c in cs], [c[2] for c in cs],
                            outs=out_bufs)
        else:
            caches[0].step(*cs[0], out=out_bufs[0])
        ci += 1

    # warm-up; the host's enqueue time per step is measured on the last ones
    host_s = []
    for i in range(args.warmup):
        torch.cuda.synchronize(dev)
        t = time.perf_counter()
        flush.zero_()
        step_all(outs)
        host_s.append(time.perf_counter() - t)
    torch.cuda.synchronize(dev)
    host_us = 1e6 * min(host_s[1:] if len(host_s) > 1 else host_s)
    # Per-kernel CUDA events on every PROF_EVERY-th timed step only: events between a
    # step's kernels stop each kernel's launch from overlapping the previous one's end
    # (programmatic dependent launch), which costs about 9% of an m2k-s1k step.
    for cache, _ in layers:
        cache.set_profiling(True)       # restart the count of profiled steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    kern_ms = []
    pairs = 0
    launches = 0
    barrier(world)
    n_prof = (steps + PROF_EVERY - 1) // PROF_EVERY
    if n_prof > 64:
        raise SystemExit(f"--steps must be <= {64 * PROF_EVERY} (per-kernel event ring)")
    with ClockSampler(local if world > 1 else 0) as clocks:
        # Steps are enqueued back to back (no host synchronisation in the timed
        # region).  A GPU sleep outside every event lets the host get ahead, so
        # the events time the kernels, not the Python loop's launch latency
        # (reported as host_us_per_step).
        sleep_s = min(2.0, 1.5 * steps * host_us * 1e-6)
        if hasattr(torch.cuda, "_sleep"):                  # a spin kernel (PyTorch's own)
            torch.cuda._sleep(int(sleep_s * 2.0e9))        # cycles at about the max SM clock
        for i in range(steps):
            for cache, _ in layers:
                cache.set_profiling(i % PROF_EVERY == 0, restart=False)
            flush.zero_()
            for cache, _ in layers:
                pairs += attn_pairs(cfg, cfg.S, cache.info()["n_valid"])
            ev[i][0].record(stream)
            step_all(outs)
            ev[i][1].record(stream)
            launches += sum(c.info()["launches"] for c, _ in layers)
        barrier(world)
    for i in range(n_prof):
        # a grouped step records its kernels' events in the first layer's ring
        kern_ms.append(caches[0].last_timings(age=n_prof - 1 - i))
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_s = max_over_ranks(sum(step_ms) / 1e3, world)
    value = aggregate_throughput(cfg.B * cfg.S * steps, world, total_s)
    attn_ms = statistics.mean(k[0] for k in kern_ms) / cfg.layers
    sel_ms = statistics.mean(k[1] for k in kern_ms) / cfg.layers
    for cache, _ in layers:
        cache.set_profiling(False)

    res = {"value": value, "ms_per_step": total_s * 1e3 / steps, "steps": steps,
           "launches": launches, "host_us": host_us, "clocks": clocks.summary(),
           "attn_ms": attn_ms, "sel_ms": sel_ms,
           "flops": 4 * cfg.d * pairs / (steps * cfg.layers)}          # per attention launch
    if with_e2e:
        # end to end through the C ABI with host buffers (pinned), copies inside the
        # region: per layer one pinned (q, k, v) set per distinct chunk, at most two
        # distinct chunks (the caches keep evolving whatever the values)
        houts = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
        e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(steps)]
        pinned = {}
        host_steps = []
        for i in range(steps):
            j = 1 + (ci + i % 2) % n_avail
            if j not in pinned:
                pinned[j] = [tuple(x.cpu().pin_memory() for x in chunks[j]) for _, chunks in layers]
            host_steps.append(pinned[j])
        h2d = sum(x.numel() * x.element_size() for hs in host_steps[0] for x in hs)
        d2h = sum(o.numel() * o.element_size() for o in houts)
        # untimed warm-up of the host-buffer path: its staging buffers are
        # allocated on first use
        for i in range(2):
            step_all(houts, host=host_steps[i % len(host_steps)])
        barrier(world)
        for i in range(steps):
            flush.zero_()
            e2e_ev[i][0].record(stream)
            step_all(houts, host=host_steps[i])
            e2e_ev[i][1].record(stream)
        barrier(world)
        e2e_s = max_over_ranks(sum(a.elapsed_time(b) for a, b in e2e_ev) / 1e3, world)
        res["e2e"] = {"value": aggregate_throughput(cfg.B * cfg.S * steps, world, e2e_s),
                      "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
        del pinned, host_steps, houts
    if with_e2e:   # the chunks the oracle's CPU baseline is timed on
        res["chunks0_host"] = [tuple(x[:1].double().cpu().numpy() for x in c) for c in layers[0][1][:8]]
    for cache, _ in layers:
        cache.close()
    del layers, outs, flush
    torch.cuda.empty_cache()
    return res


def roofline_objects(cfg, res, peaks):
    achieved = res["flops"] / (res["attn_ms"] * 1e-3) / 1e12
    sel_bytes = select_scatter_bytes(cfg, cfg.S)
    sel_gbs = sel_bytes / (res["sel_ms"] * 1e-3) / 1e9
    # a multi-layer step keeps the GPU busy for tens of milliseconds per step,
    # back to back: its attention runs at the power-capped sustained clock, so
    # it is read against the sustained GEMM peak; a single layer's steps are
    # short and read against the burst peak
    sustained = cfg.layers > 1 and peaks.get("bf16_tflops_sustained")
    peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    return (
        {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
         "frac": achieved / peak, "frac_of_burst_peak": achieved / peaks["bf16_tflops"],
         "traffic": traffic_for(cfg),
         "kernel": "attention + summed weights",
         "peak_source": f"{peaks['source']} bf16 dense ({'sustained' if sustained else 'burst'})",
         "algorithmic_flops_per_launch": res["flops"], "ms_per_launch": res["attn_ms"]},
        {"bound": "hbm", "achieved": sel_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
         "frac": sel_gbs / peaks["hbm_gbs"], "kernel": "tail: score accumulate + select + scatter",
         "peak_source": f"{peaks['source']} copy bandwidth",
         "algorithmic_bytes_per_launch_set": sel_bytes, "ms_per_launch_set": res["sel_ms"]})


def run_ours(args, cfg):
    world, rank, local = dist_setup(args.gpus)
    wl = workload_module()
    peaks = load_peaks()
    res = measure(args, cfg, world, rank, local, args.steps, with_e2e=True)
    roof, roof_sel = roofline_objects(cfg, res, peaks)
    line = {
        "metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if cfg.dtype == torch.bfloat16 else "f32", "data": "synthetic",
        "config": config_dict(cfg, world),
        "roofline": roof,
        "roofline_select_scatter": roof_sel,
        "e2e": res["e2e"],
        "gpu_launches": res["launches"],
        "host_us_per_step": res["host_us"],
        "clocks": res["clocks"],
        "kernel_ms_per_layer": {"attention": res["attn_ms"],
                                "tail (score accumulate + select + scatter)": res["sel_ms"]},
        "kernel_events": f"CUDA events around each kernel on every {PROF_EVERY}th timed step",
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, desc, n, el = oracle_sample(cfg, res["chunks0_host"], budget_s=args.cpu_budget)
        cores = host_cores()
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": cores["blas_threads"],
                                "os_cpu_count": cores["os_cpu_count"], "kind": "oracle",
                                "sample": desc}
    # the other full-size single-layer workloads: their roofline figures
    if not args.no_extra and args.config == 4:
        other = {}
        for cid in (2, 3):
            c2 = wl.CONFIGS[cid]
            r2 = measure(args, c2, world, rank, local, min(args.steps, 24), with_e2e=False)
            ro, rs = roofline_objects(c2, r2, peaks)
            other[c2.name] = {"workload": f"{c2.name}: {c2.describe()}", "value": r2["value"],
                              "unit": UNIT, "steps": r2["steps"], "ms_per_step": r2["ms_per_step"],
                              "roofline": ro, "roofline_select_scatter": rs,
                              "gpu_launches": r2["launches"], "clocks": r2["clocks"]}
        line["other_workloads"] = other
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# the sources each attention path is built from: a traffic figure stays valid
# while none of them changes
KERNEL_SOURCES = {
    "fused": ["attn_umma.cu", "attn_common.cuh", "sm100.cuh", "h2o_internal.cuh"],
    "stream": ["attn_stream.cu", "attn_common.cuh", "sm100.cuh", "h2o_internal.cuh"],
}


def sources_sha(names):
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "h2o_kv_cache_b200", "csrc")
    for n in sorted(names):
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(n.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", type=int, default=4)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the 16k- and 32k-slot workloads measured after the default one")
    ap.add_argument("--layers", type=int, default=None,
                    help="run only this many of the workload's layers (a smaller case for profilers)")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--clock-poller", type=int, default=None, help=argparse.SUPPRESS)
    args = ap.parse_args()
    if args.clock_poller is not None:
        clock_poller(args.clock_poller)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    cfg = workload_module().CONFIGS[args.config]
    if args.layers is not None:
        import dataclasses
        cfg = dataclasses.replace(cfg, layers=max(1, min(args.layers, cfg.layers)))
    if args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
