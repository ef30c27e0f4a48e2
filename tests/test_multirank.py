"""The multi-rank bench logic on CPU: two gloo ranks, as under torchrun with --gpus 2.

bench.py runs one replica of the layer stream per GPU (the path does not shard at this size), so
the only cross-rank steps are the barrier around the timed region, the max of the timings over
ranks and the whole-job aggregate; the reference arm runs on rank 0 alone.  These run here with
the gloo backend on 127.0.0.1 (no GPU needed).
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist                           # noqa: E402
import torch.multiprocessing as mp                         # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        # rank r times (r + 1) s for the kernel steps and 3 (r + 1) s end to end
        secs, secs_e2e = bench.max_over_ranks(dist, [1.0 * (rank + 1), 3.0 * (rank + 1)], "cpu")
        value = bench.whole_job_gbps(1e9, 10, secs, world)
        dist.barrier()
        q.put((rank, secs, secs_e2e, value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_whole_job_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, secs, secs_e2e, value in out:
        assert secs == 2.0 and secs_e2e == 6.0           # the slowest rank bounds both timings
        assert value == pytest.approx(1e9 * 10 * 2 / 2.0 / 1e9)   # both ranks' bytes over the max time


def test_whole_job_value_single_rank():
    import bench
    assert bench.whole_job_gbps(7_725_072, 73, 73 * 23.4e-6, 1) == pytest.approx(7_725_072 / 23.4e-6 / 1e9)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import argparse

    import bench
    args = argparse.Namespace(steps=1, warmup=1, gpus=2)
    assert bench.run_reference(args, 1, 2) == 0          # rank 1: exits 0 without work
    assert capsys.readouterr().out == ""
