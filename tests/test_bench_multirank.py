"""The multi-rank path of bench.py on CPU: two gloo ranks, each with its own
batch (its own routing group) and the same expert weights; timings are
aggregated by their maximum and throughput counts every rank's tokens."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from switch_inputs import TINY


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = TINY.with_(T=64)
        inp = bench.host_inputs(wl, rank)
        t_ms = [12.5, 20.0][rank]                       # rank 1 is the slow one
        m = bench.max_over_ranks(t_ms, torch.device("cpu"), world)
        v = bench.job_throughput(wl.T, 10, world, m)
        digest = torch.tensor([float(inp.x.sum()), float(inp.w1.sum())], dtype=torch.float64)
        allx = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(allx, digest)
        out[rank] = (m, v, [a.tolist() for a in allx])
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    for rank in range(world):
        m, v, digests = out[rank]
        assert m == 20.0                                 # the slowest rank's time
        assert v == pytest.approx(64 * 10 * 2 / 0.020)   # all ranks' tokens
        (x0, w0), (x1, w1) = digests
        assert x0 != x1                                  # each rank its own batch
        assert w0 == w1                                  # same expert weights


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.25, torch.device("cpu"), 1) == 3.25
    assert bench.job_throughput(1000, 4, 1, 2.0) == pytest.approx(2e6)
