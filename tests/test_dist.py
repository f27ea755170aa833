"""The multi-rank host logic of bench.py on CPU: gloo, world size 2.

Ranks run independent copies of the parameter set (the blocks need no data
exchange), so the only cross-rank step is the job time, the max over ranks,
and the whole-job throughput built from it.  The reference arm runs on rank 0
alone; other ranks exit without work.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    ms = 10.0 + 5.0 * rank
    job = bench.max_over_ranks(ms, dist, torch.device("cpu"))
    val = bench.job_tflops(1e12, world, job)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, job, val))


@pytest.mark.parametrize("world", [2])
def test_job_time_is_max_over_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, job, val in out:
        assert job == 15.0                       # the slower rank's time
        assert abs(val - 2 * 1e12 / 15e-3 / 1e12) < 1e-9


def test_reference_arm_other_ranks_exit_quietly(capsys):
    import argparse
    import bench
    from shampoo_second_order_b200 import workloads as wl
    args = argparse.Namespace(steps=1, warmup=0, config="single_64x32")
    assert bench.reference_arm(args, wl.CONFIGS["single_64x32"], rank=1, world=2) == 0
    assert capsys.readouterr().out == ""


def test_single_process_needs_no_collective():
    import bench
    assert bench.max_over_ranks(7.5, None, None) == 7.5
