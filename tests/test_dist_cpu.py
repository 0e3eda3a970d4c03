"""Multi-rank host logic of bench.py on CPU: two gloo ranks.

The attention path shards over independent (b, h) problems with no exchange
step, so the only cross-rank logic is the timing: every rank reports its own
time, the job takes as long as the slowest rank, and the whole-job value
counts every rank's work (weak scaling)."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, ms, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(ms[rank], world)
        val = bench.weak_scaling_value(1e12, got, world)
        out[rank] = (got, val)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_value_two_gloo_ranks():
    world = 2
    ms = [3.0, 5.0]
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, ms, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(world):
        got, val = out[r]
        assert got == 5.0
        # 2 ranks x 1 TFLOP each in 5 ms
        assert val == pytest.approx(2 * 1e12 / 5e-3 / 1e12)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(4.5, 1) == 4.5
    assert bench.weak_scaling_value(2e12, 4.0, 1) == pytest.approx(500.0)
