"""The multi-rank path of bench.py on CPU: two gloo ranks (no GPU).

bench.py runs one decode stream per rank (weak scaling, no data-path
collective); the only cross-rank steps are the barriers around the timed
region and the max over ranks of the device time.  These tests drive those
helpers, the whole-job throughput and the rank-0-only reference arm with a
world of two processes on the host.
"""
import json
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out_dir: str):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench  # noqa: E402
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # each rank reports a different device time; all must see the max
        mine = 0.25 + 0.5 * rank
        bench.barrier(world)
        t = bench.max_over_ranks(mine, world)
        value = bench.job_throughput(1e9, 10, world, t)
        # the reference arm prints on rank 0 only, and returns at once elsewhere
        args = type("A", (), dict(warmup=0, steps=1, ref_seconds=0.0, gpus=world))()
        import contextlib
        import io
        buf = io.StringIO()
        if rank != 0:
            with contextlib.redirect_stdout(buf):
                bench.run_reference(args, world, rank)
        bench.barrier(world)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"t": t, "value": value, "ref_stdout": buf.getvalue()}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_the_max_time_and_the_job_value(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["t"] == pytest.approx(0.75)
        # 1 GB per step per rank, 10 steps, 2 ranks, 0.75 s -> 26.67 GB/s
        assert r["value"] == pytest.approx(1e9 * 10 * 2 / 0.75 / 1e9)
    assert res[1]["ref_stdout"] == ""


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1.5, 1) == 1.5
    bench.barrier(1)
    assert bench.job_throughput(2e9, 5, 1, 2.0) == pytest.approx(5.0)
