"""The multi-GPU bench path on CPU: two gloo ranks, each timing its own
replica; the job time is the slowest rank and the value is the whole-job
throughput.  No GPU and no data-path collective are involved."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, times, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        t = bench.max_over_ranks(times[rank], world)
        out[rank] = (t, bench.whole_job_tflops(1e12, 10, world, t))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_whole_job_throughput():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    times = [120.0, 150.0]  # ms for 10 steps on each rank
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, times, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(2):
        t, v = out[r]
        assert t == 150.0
        # 2 ranks x 10 steps x 1e12 FLOP in 0.15 s
        assert abs(v - 2 * 10 * 1e12 / 0.15 / 1e12) < 1e-9


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_tflops(2e12, 4, 1, 1000.0) == pytest.approx(8.0)
