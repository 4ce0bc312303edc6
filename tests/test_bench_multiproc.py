"""Host logic of bench.py across ranks, on CPU with the gloo backend and two processes:
the barrier, the max over ranks of the step time, the whole-job throughput, and that
only rank 0 runs the oracle arm."""
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


def _worker(rank, world, port, out):
    import argparse
    from datetime import timedelta

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        bench.barrier(world)
        step_ms = 1.0 + 2.0 * rank                       # rank 1 is the slow one
        m = bench.max_over_ranks(step_ms, world)
        value = bench.whole_job_value(1e12, m, world)
        args = argparse.Namespace(steps=1, warmup=0)
        ref = bench.run_reference(args, world, rank) if rank != 0 else "skipped"
        bench.barrier(world)
        out.put((rank, m, value, ref))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_reporting():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    codes = [p.exitcode for p in procs]
    assert codes == [0, 0], codes
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, m, value, ref in res:
        assert m == pytest.approx(3.0)                  # max over ranks, on every rank
        assert value == pytest.approx(2 * 1e12 / 3e-3 / 1e12)
    assert res[1][3] is None                            # rank 1 does no oracle work


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.5, 1) == 4.5
    assert bench.whole_job_value(2e12, 1.0, 1) == pytest.approx(2000.0)
