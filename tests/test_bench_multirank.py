"""The benchmark's multi-rank host logic, on CPU: two gloo ranks.

bench.py --gpus N runs one process per GPU, each with its own layer (no
data-path collective).  What crosses ranks is the timing: every rank times its
region, the slowest rank's time is taken (all_reduce MAX), and the whole-job
value is all ranks' bytes over that time.  These tests run that logic over a
world-size-2 gloo group on the host; no GPU is touched.
"""
from __future__ import annotations

import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, outdir: str):
    import datetime
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # Each rank's own region time; every rank must end up with the slowest.
        mine = [1.25, 3.5][rank]
        slowest = bench.max_over_ranks(dist, mine, "cpu")
        dist.barrier()
        # Non-zero ranks of the reference arm return at once and print nothing.
        printed = ""
        if rank != 0:
            buf = io.StringIO()
            args = type("A", (), dict(q=3, batch=1, warmup=3, steps=2, ref_rows=32))()
            with redirect_stdout(buf):
                ret = bench.run_reference(args)
            assert ret is None
            printed = buf.getvalue()
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump({"slowest": slowest, "seed": bench.rank_seed(rank), "printed": printed}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert [r["slowest"] for r in res] == [3.5, 3.5]
    assert res[0]["seed"] != res[1]["seed"]          # independent layers per rank
    assert res[1]["printed"] == ""                   # only rank 0 prints a line


def test_aggregate_is_all_ranks_bytes_over_the_slowest_time():
    sys.path.insert(0, ROOT)
    import bench
    # 765,052,928 B per step, 200 steps, 2 ranks, slowest rank 30 ms:
    # 2 * 200 * 765,052,928 B / 0.030 s = 10,200.7 GB/s.
    v = bench.aggregate_gbs(765_052_928, 200, 2, 30.0)
    assert v == pytest.approx(2 * 200 * 765_052_928 / 0.030 / 1e9)
    assert bench.aggregate_gbs(765_052_928, 200, 1, 30.0) == pytest.approx(v / 2)
    assert bench.max_over_ranks(None, 2.5, "cpu") == 2.5
