"""Replicas across GPUs: the host logic of bench.py's N > 1 path on CPU (gloo, two ranks).

The layer has no exchange step, so N GPUs run N independent replicas; the only
collective is the max over ranks of the step timings.  These tests run that reduction
and the whole-job throughput with world size 2 on the gloo backend."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r reports step times (1 + r) ms and e2e (3 - r) ms: the max is taken per entry
        ms, e2e = bench.max_over_ranks([1.0 + rank, 3.0 - rank], world, torch.device("cpu"))
        out[rank] = (ms, e2e, bench.job_tokens_per_s(world, 32, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        ms, e2e, v = res[r]
        assert ms == 2.0 and e2e == 3.0
        assert v == pytest.approx(2 * 32 / 2e-3)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks([1.5, 2.5], 1, torch.device("cpu")) == [1.5, 2.5]
    assert bench.job_tokens_per_s(1, 32, 0.366) == pytest.approx(32 / 0.366e-3)
