"""bench.py's multi-rank host logic on the CPU: two gloo ranks.

The path runs as independent replicas (no data-path collective); the only
cross-rank steps are the barrier around the timed region and the reduction of
the timing: value = units of all ranks / the slowest rank's time.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, lr = bench.dist_setup(world)
        assert (w, r, lr) == (world, rank, rank)
        bench.barrier(world)
        local_time = [2.0, 3.0][rank]
        local_units = [100.0, 300.0][rank]
        value, t = bench.aggregate(local_time, local_units, world, torch.device("cpu"))
        q.put((rank, value, t))
        # the reference arm: rank 0 alone works; other ranks return at once
        if rank == 1:
            class A:
                steps, warmup, gpus = 1, 1, world
            assert bench.run_reference(A, world, rank) is None
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_max_time_and_summed_units():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, value, t in res:
        assert t == pytest.approx(3.0)
        assert value == pytest.approx(400.0 / 3.0)


def test_world_size_mismatch_is_rejected(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "1")
    with pytest.raises(SystemExit):
        bench.dist_setup(2)
