"""The bench's multi-rank plumbing on the CPU: two gloo ranks.

The hot path shards into independent replicas (one per GPU, no data-path
collective), so what runs across ranks is only the timing plumbing: the
process group, the barrier, the max over ranks of the timed interval and the
whole-job throughput built from it, and the reference arm's rank-0-only
rule.  These run here as two processes on the gloo backend.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    args = bench.parse_args(["--gpus", str(world), "--steps", "4", "--warmup", "3"])
    w, r, local = bench.dist_setup(args)
    try:
        assert dist.get_backend() == "gloo"
        bench.barrier()
        # each rank timed a different interval; every rank sees the slowest
        mine = 10.0 + 5.0 * r
        slowest = bench.dist_max(mine, torch.device("cpu"))
        value = bench.aggregate_rate(1000, 4, w, slowest)
        # the reference arm: only rank 0 does any work
        ref = None
        if r != 0:
            ref = bench.run_reference(args, w, r)
        out[r] = (w, r, slowest, value, ref)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_aggregate():
    world, port = 2, _free_port()
    # spawn, not fork: earlier tests may have started the oracle's threads
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    assert sorted(out.keys()) == [0, 1]
    for r in range(world):
        w, rank, slowest, value, ref = out[r]
        assert (w, rank) == (world, r)
        assert slowest == 15.0                 # max over ranks, on every rank
        # 1000 units per step, 4 steps, 2 ranks, 15 ms -> 533,333 units/s
        assert value == pytest.approx(1000 * 4 * 2 / 0.015)
    assert out[1][4] is None                   # rank 1 of the reference arm idles


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    assert not dist.is_initialized()
    assert bench.dist_max(3.5, torch.device("cpu")) == 3.5
    bench.barrier()
    assert bench.aggregate_rate(10, 5, 1, 1000.0) == pytest.approx(50.0)
