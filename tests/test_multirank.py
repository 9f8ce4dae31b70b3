"""Host logic of the multi-rank benchmark on CPU (gloo, world size 2).

The layer shards by tokens with replicated weights, so ranks exchange no data:
each rank draws its own tokens (rank-dependent seed) against the same weights,
and the only cross-rank step is the max-over-ranks reduction of the timings,
from which the whole-job tokens/s is formed.
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


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_layer_logits_b200 import workloads as wl

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = wl.custom("mr", 4, 16, 2, 128, 128)
        logits = wl.make_logits(w, seed=bench.rank_seed(0, rank))
        w13, w2 = wl.make_weights(w, seed=0)
        gathered = [torch.empty_like(logits) for _ in range(world)]
        dist.all_gather(gathered, logits)
        digests = [torch.empty(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(digests, torch.tensor([float(w13.float().sum() + w2.float().sum())],
                                              dtype=torch.float64))
        local_ms = 1.0 + rank  # rank 1 is the slower one
        slowest = bench.max_over_ranks(local_ms, dist, "cpu")
        out[rank] = dict(slowest=slowest,
                         distinct_tokens=not torch.equal(gathered[0], gathered[1]),
                         same_weights=bool(digests[0].item() == digests[1].item()),
                         value=bench.weak_scaling_value(world, w.T, slowest))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    assert set(out.keys()) == {0, 1}
    for r in range(world):
        assert out[r]["slowest"] == 2.0          # max over ranks, seen by every rank
        assert out[r]["distinct_tokens"]
        assert out[r]["same_weights"]
        assert out[r]["value"] == pytest.approx(2 * 4 / 2e-3)


def test_single_rank_helpers():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.rank_seed(0, 0) != bench.rank_seed(0, 1)
    assert bench.weak_scaling_value(1, 8, 0.125) == pytest.approx(64000.0)


def test_step_stats():
    sys.path.insert(0, ROOT)
    import bench

    st = bench.step_stats([float(v) for v in range(1, 11)], lambda v: v)
    assert st == {"median": 5.5, "p10": 1.9, "p90": 9.1}
    assert bench.step_stats([0.25], lambda v: v) == {"median": 0.25, "p10": 0.25, "p90": 0.25}
    # every statistic goes through the max-over-ranks reduction
    assert bench.step_stats([1.0, 3.0], lambda v: v + 100)["median"] == 102.0
