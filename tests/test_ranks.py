"""The multi-rank bench path on CPU: two gloo ranks agree on the slowest rank's time, the
whole-job value counts every rank's chunk, and the reference arm runs on rank 0 only."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        slowest = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")
        q.put((rank, slowest))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert got == [(0, 15.0), (1, 15.0)]


def test_whole_job_value_counts_every_rank():
    import bench
    one = bench.whole_job_tflops(1e12, 1, 2.0)
    assert one == pytest.approx(500.0)
    assert bench.whole_job_tflops(1e12, 4, 2.0) == pytest.approx(4 * one)
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import argparse
    import bench
    bench.run_reference(argparse.Namespace(config="1", steps=1, warmup=0), rank=1)
    assert capsys.readouterr().out == ""
