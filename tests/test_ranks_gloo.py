"""The multi-rank bench plumbing on CPU with two gloo ranks (no GPU).

bench.py runs one replica per rank on its own batch (the (b, h) problems are
independent, so there is no data-path collective). The only communication is the
max-over-ranks reduction of the timings; these tests check it and the whole-job
throughput, plus that the ranks' batches differ.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import bench
    from entmax_sm_attention_b200.workloads import make_inputs, small_case

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 30.0][rank]
        mx = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        value = bench.job_throughput(world, 8192, 10, mx)
        q = make_inputs(small_case("r", L=64), seed=bench.rank_seed(0, rank))["Q"]
        sums = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(sums, q.float().sum().reshape(1))
        out[rank] = (mx, value, [float(x) for x in sums])
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
        res = dict(out)
    for rank in range(world):
        mx, value, sums = res[rank]
        assert mx == 30.0                                 # the slowest rank
        assert value == pytest.approx(2 * 8192 * 10 / 0.030)
        assert sums[0] != sums[1]                         # independent batches


def test_single_rank_needs_no_process_group():
    import bench

    assert bench.max_over_ranks(7.0, 1, torch.device("cpu")) == 7.0
    assert bench.job_throughput(1, 100, 4, 2.0) == pytest.approx(200000.0)
