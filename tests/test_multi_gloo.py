"""Multi-process (world_size 2, gloo, CPU) tests of the replicas-only multi-GPU
host path: unit sharding and the max-over-ranks step time."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from decode_kv_cache_eviction_b200 import shard
from decode_kv_cache_eviction_b200 import workloads as W


@pytest.mark.parametrize("redundancy", ["gemm", "closed"])
def test_shard_units_partition_and_balance(redundancy):
    n = W.unit_lengths(W.WORKLOADS["ragged_serving"], 0)
    cost = shard.unit_cost(n, redundancy)
    for world in (1, 2, 3, 8):
        parts = shard.shard_units(n, world, redundancy)
        allu = np.sort(np.concatenate(parts))
        np.testing.assert_array_equal(allu, np.arange(len(n)))
        loads = np.array([cost[p].sum() for p in parts])
        # greedy LPT: no rank exceeds another by more than the costliest unit
        assert loads.max() - loads.min() <= cost.max()
        for p in parts:
            assert np.all(np.diff(p) > 0)


def test_gemm_sharding_balances_the_quadratic_work():
    """Units of 2K-8K tokens: balancing N alone can leave the N^2 GEMM work
    uneven; the GEMM cost model keeps it within a few percent."""
    rng = np.random.default_rng(0)
    n = np.concatenate([np.full(40, 8192), np.full(160, 2048)])
    rng.shuffle(n)
    for world in (2, 4, 8):
        parts = shard.shard_units(n, world, "gemm")
        quad = np.array([(n[p].astype(np.float64) ** 2).sum() for p in parts])
        assert quad.max() / quad.mean() < 1.05


def test_sub_offsets_and_rows():
    off = np.array([0, 5, 5, 12, 20])
    units = np.array([3, 0, 2])
    np.testing.assert_array_equal(shard.sub_offsets(off, units), [0, 8, 13, 20])
    rows = shard.gather_rows(off, units)
    np.testing.assert_array_equal(rows, list(range(12, 20)) + list(range(0, 5)) + list(range(5, 12)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        n = W.unit_lengths(W.WORKLOADS["ragged_serving"], 3)
        mine = shard.shard_units(n, world)[rank]
        got = [None] * world
        dist.all_gather_object(got, mine.tolist())
        # each rank's local "step time"; the reported time is the max over ranks
        t = torch.tensor([float(n[mine].sum()) / 1e6], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        q.put((rank, got, float(t.item()), float(n[mine].sum()) / 1e6))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_sharding_covers_all_units_once():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=100) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    gathered = res[0][1]
    assert res[1][1] == gathered
    allu = sorted(u for part in gathered for u in part)
    n_units = W.WORKLOADS["ragged_serving"].num_units
    assert allu == list(range(n_units))
    tmax = max(r[3] for r in res)
    assert all(abs(r[2] - tmax) < 1e-12 for r in res)
