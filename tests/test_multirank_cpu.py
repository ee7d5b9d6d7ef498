"""The benchmark's multi-rank paths on CPU: gloo, world size 2, two processes.

Replicas: each rank runs an independent layer (weak scaling).  Head sharding: the ranks
split one layer by whole KV groups (strong scaling).  Either way the only cross-rank
operations are the barrier and the max-over-ranks reduction of the timings, which these
tests exercise with the same functions bench.py uses."""
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


def _shard_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    import long_context_prefill_estimate_b200 as rr

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        H, Hkv = 28, 4
        shard = rr.head_shard(rank, world, H, Hkv)
        got = [None] * world
        dist.all_gather_object(got, shard)
        ms = bench.max_over_ranks(20.0 - 4.0 * rank)      # rank 0 is the slower one
        q.put((rank, got, ms, bench.aggregate_tflops(1, 1e12, ms),
               bench.config_dict(__import__("workloads").get(4), world, "heads")["parallelism"]))
    finally:
        dist.destroy_process_group()


def test_two_rank_head_sharding():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, shards, ms, value, par in out:
        # contiguous whole KV groups, disjoint, covering the layer
        assert shards == [(0, 14, 0, 2), (14, 28, 2, 4)]
        assert ms == 20.0
        assert value == pytest.approx(1e12 / 20e-3 / 1e12)   # one layer in all, strong scaling
        assert par.startswith("heads2")


def test_head_shard_map():
    sys.path.insert(0, ROOT)
    import long_context_prefill_estimate_b200 as rr

    for H, Hkv in [(32, 8), (28, 4), (8, 8), (14, 2)]:
        for world in range(1, Hkv + 1):
            parts = [rr.head_shard(r, world, H, Hkv) for r in range(world)]
            assert parts[0][0] == 0 and parts[0][2] == 0
            assert parts[-1][1] == H and parts[-1][3] == Hkv
            for (a0, a1, b0, b1), (c0, c1, e0, e1) in zip(parts, parts[1:]):
                assert a1 == c0 and b1 == e0            # contiguous and disjoint
            for h0, h1, g0, g1 in parts:
                assert g1 > g0 and (h0, h1) == (g0 * H // Hkv, g1 * H // Hkv)
                assert abs((g1 - g0) - Hkv / world) < 1   # as even as the groups divide
    with pytest.raises(ValueError):
        rr.head_shard(0, 3, 4, 2)       # more ranks than KV groups
    with pytest.raises(ValueError):
        rr.head_shard(2, 2, 8, 2)
    with pytest.raises(ValueError):
        rr.head_shard(0, 1, 6, 4)
