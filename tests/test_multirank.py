"""Multi-rank host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

The path has no exchange step, so N GPUs run N independent replicas; what
crosses ranks is only timing.  These tests check that each rank draws its own
batch, that the step time every rank reports is the slowest rank's, and that
the job throughput counts every rank's units over that time.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from learned_token_indexer_b200 import workloads as W


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        step_ms = [3.0, 5.0][rank]                         # rank 1 is slower
        slowest = bench.max_over_ranks(step_ms, torch.device("cpu"))
        w = bench.rank_workload(W.PREFILL, rank)
        out[rank] = (slowest, w.seed, bench.job_throughput(world, 8192, slowest))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_the_slowest_time_and_own_batches():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 5.0                   # max over ranks
    assert res[0][1] != res[1][1]                          # independent batches
    assert res[0][1] == W.PREFILL.seed                     # rank 0 keeps the workload's seed
    assert res[0][2] == pytest.approx(2 * 8192 / 5e-3)     # all ranks' rows over the slowest time


def test_single_process_is_the_identity():
    assert bench.max_over_ranks(7.5, torch.device("cpu")) == 7.5
    assert bench.rank_workload(W.DECODE, 0) is W.DECODE
    assert bench.job_throughput(1, 64, 2.0) == pytest.approx(32000.0)
