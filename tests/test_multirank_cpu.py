"""The N > 1 path of bench.py on the CPU: two ranks over gloo.

bench.py runs one process per GPU, with no collective on the data path
(weak scaling).  Its multi-rank logic is small: every time is reduced to
the slowest rank's, the whole-job throughput multiplies the per-rank bytes
by the world size, and the reference arm runs on rank 0 alone.  These tests
run that logic in two spawned gloo ranks on 127.0.0.1."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.join(os.path.dirname(__file__), "..")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [0.0571, 0.0604][rank]            # per-rank step times
        ms_max = bench.reduce_max(ms, dist, "cpu")
        val = bench.job_throughput(world, 268_435_456, ms_max)
        # the reference arm: rank 0 alone runs the oracle; others return at once
        skipped = None
        if rank != 0:
            class A:
                steps, warmup, gpus = 1, 0, world
            bench.run_reference(A(), rank)
            skipped = True
        out[rank] = (ms_max, val, skipped)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_weak_scaling_value():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert set(res) == {0, 1}
    for rank in (0, 1):
        ms_max, val, _ = res[rank]
        assert ms_max == pytest.approx(0.0604)             # the slowest rank's time
        assert val == pytest.approx(2 * 268_435_456 / 0.0604e-3 / 1e9)
    assert res[1][2] is True                               # rank 1 skipped the reference arm


def test_reduce_max_without_group_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.25) == 3.25
    assert bench.job_throughput(1, 1e9, 1000.0) == pytest.approx(1.0)
