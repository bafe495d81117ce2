"""Replica logic of N-GPU runs, as world-size-2 gloo process groups on CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from h2o_kv_cache_b200.replicas import (aggregate_throughput, max_over_ranks,
                                               replica_stream_layer)
        from h2o_kv_cache_b200.workload import CONFIGS, gen_sequence
        # each replica times its own work; the run's time is the slowest replica's
        my_time = 1.0 + rank
        t = max_over_ranks(my_time, world, device="cpu")
        cfg = CONFIGS[0]
        Q, _, _ = gen_sequence(cfg, 0, replica_stream_layer(rank, 0), T=64)
        gathered = [torch.zeros_like(Q) for _ in range(world)]
        dist.all_gather(gathered, Q)
        q.put((rank, t, aggregate_throughput(100.0, world, t),
               all(torch.equal(gathered[i], gathered[j]) for i in range(world)
                   for j in range(world) if i != j)))
    finally:
        dist.destroy_process_group()


def test_replicas_time_is_the_slowest_rank_and_streams_differ():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, thr, same in res:
        assert t == 2.0                      # max over ranks of 1.0, 2.0
        assert thr == pytest.approx(100.0)   # 100 units per rank x 2 ranks / 2 s
        assert not same                      # replicas run different seeded streams
    # single-process form needs no group
    from h2o_kv_cache_b200.replicas import max_over_ranks
    assert max_over_ranks(3.5, 1) == 3.5
