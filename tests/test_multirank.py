"""The multi-GPU host logic of bench.py (replicas: one process per GPU, no
data-path exchange) with world_size 2 over gloo on the CPU: per-rank
workloads, the max-over-ranks timing and the whole-job throughput."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = [3.0, 5.0][rank]  # rank 1 is the slower one
        worst = bench.max_over_ranks(ms, dist, "cpu")
        wl = bench.rank_workload("decode1m", rank)
        out[rank] = (worst, wl.seed, wl.batch, bench.tokens_per_s(wl.batch, world, worst))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_over_gloo():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    (w0, s0, b0, v0), (w1, s1, b1, v1) = out[0], out[1]
    assert w0 == w1 == 5.0, "every rank sees the slowest rank's time"
    assert s0 != s1 and b0 == b1, "replicas: same shapes, own inputs"
    assert v0 == v1 == pytest.approx(b0 * 2 / 5e-3)


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(7.5, None, "cpu") == 7.5
    assert bench.rank_workload("decode1m", 0).seed == bench.rank_workload("decode1m", 0).seed
    assert bench.tokens_per_s(4, 1, 100.0) == pytest.approx(40.0)
