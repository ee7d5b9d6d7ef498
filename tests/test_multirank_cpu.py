"""The benchmark's multi-rank path on CPU: gloo, world size 2, two processes.

Each rank runs an independent layer (weak scaling); the only cross-rank operations are the
barrier and the max-over-ranks reduction of the timings, which these tests exercise with the
same functions bench.py uses."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slower one
        dist.barrier()
        ms = bench.max_over_ranks(local_ms)
        e2e_ms = bench.max_over_ranks(3.0 - rank)
        value = bench.aggregate_tflops(world, 1e12, ms)
        q.put((rank, ms, e2e_ms, value, bench.dist_env()))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_weak_scaling_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, e2e_ms, value, env in out:
        assert ms == 15.0 and e2e_ms == 3.0
        assert value == pytest.approx(world * 1e12 / 15e-3 / 1e12)
        assert env == (rank, world, rank)


def test_single_process_without_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(7.5) == 7.5
    assert bench.aggregate_tflops(1, 2e12, 1000.0) == pytest.approx(2.0)
