"""Tensor-parallel host logic on the CPU: shard plans, shard slicing and the
collectives, over gloo process groups of 2 and 3 ranks.

Each rank's product is the FP64 oracle on its own shard (a test stands it in
for the GPU library); the exchanged result must equal the oracle on the whole
matrix.  No GPU is touched.
"""
from __future__ import annotations

import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from weight_only_quantized_bcq_b200 import sharded as T  # noqa: E402


# ---------------------------------------------------------------------------
# Plans (no process group)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("m,world", [(1, 1), (31, 2), (32, 2), (100, 3), (4096, 8), (300, 4), (65, 3)])
def test_row_plans_partition_the_rows_in_tiles(m, world):
    plans = [T.plan_rows(m, 256, 3, 128, world, r) for r in range(world)]
    assert plans[0].lo == 0 and plans[-1].hi == m
    for a, b in zip(plans, plans[1:]):
        assert a.hi == b.lo                                   # contiguous, no overlap
    for p in plans:
        assert p.lo % T.ROW_ALIGN == 0 or p.lo == m           # every range starts on a tile (or is empty)
        assert p.hi == m or p.hi % T.ROW_ALIGN == 0
        assert p.span >= max(q.hi - q.lo for q in plans)
        assert p.local_m == p.hi - p.lo and p.local_n == 256
    sizes = [-(-(p.hi - p.lo) // T.ROW_ALIGN) for p in plans]
    assert max(sizes) - min(sizes) <= 1                       # balanced to one tile


@pytest.mark.parametrize("n,g,world", [(1024, 128, 2), (12288, 128, 8), (640, 64, 3), (256, 256, 1), (512, 8, 5)])
def test_input_plans_partition_whole_groups(n, g, world):
    plans = [T.plan_inputs(64, n, 2, g, world, r) for r in range(world)]
    assert plans[0].lo == 0 and plans[-1].hi == n
    for a, b in zip(plans, plans[1:]):
        assert a.hi == b.lo
    for p in plans:
        assert p.lo % g == 0 and p.hi % g == 0
        assert p.local_n == p.hi - p.lo and p.local_m == 64
    sizes = [(p.hi - p.lo) // g for p in plans]
    assert max(sizes) - min(sizes) <= 1
    assert plans[0].span == max(sizes) * g


def test_plans_reject_bad_arguments():
    with pytest.raises(ValueError):
        T.plan_rows(64, 64, 1, 8, 2, 2)
    with pytest.raises(ValueError):
        T.plan_inputs(64, 100, 1, 64, 2, 0)
    with pytest.raises(ValueError):
        T.plan_paired(100, 64, 64, 1, 64, 2, 0)


def test_take_shard_slices_signs_and_scales():
    q, m, n, g = 2, 70, 256, 64
    signs = torch.arange(q * m * n, dtype=torch.int32).reshape(q, m, n)
    alpha = torch.arange(q * (n // g) * m, dtype=torch.int32).reshape(q, n // g, m)
    pr = T.plan_rows(m, n, q, g, 2, 1)
    s, a = T.take_shard(pr, signs, alpha)
    assert torch.equal(s, signs[:, pr.lo:pr.hi]) and torch.equal(a, alpha[:, :, pr.lo:pr.hi])
    pi = T.plan_inputs(m, n, q, g, 3, 1)
    s, a = T.take_shard(pi, signs, alpha)
    assert torch.equal(s, signs[:, :, pi.lo:pi.hi])
    assert torch.equal(a, alpha[:, pi.lo // g:pi.hi // g])
    x = torch.arange(3 * n).reshape(3, n)
    assert torch.equal(T.take_input_slice(pi, x), x[:, pi.lo:pi.hi])
    assert T.take_input_slice(pr, x) is x


def test_paired_plans_cover_the_same_range():
    for world in (1, 2, 3, 4):
        for r in range(world):
            a, b = T.plan_paired(1024, 512, 256, 3, 128, world, r)
            assert a.kind == "rows" and b.kind == "inputs"
            assert (a.lo, a.hi) == (b.lo, b.hi) and a.lo % 128 == 0


# ---------------------------------------------------------------------------
# Collectives over gloo, with the oracle as each rank's product
# ---------------------------------------------------------------------------
def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(q, m, n, g, batch, seed):
    import bcq_synth as S
    gen = S.generator(seed)
    signs = S.draw_signs(gen, q, m, n)
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02)
    x = S.draw_x(gen, batch, n)
    return signs, alpha, x


def _oracle(x, signs, alpha, g):
    from oracle import bcq_oracle as O
    return torch.from_numpy(O.bcq_matmul(x.numpy(), signs.numpy(), alpha.numpy(), g))


def _rank_main(rank, world, port, outdir):
    import datetime
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        res = {}
        q, m, n, g, batch = 3, 200, 640, 64, 3
        signs, alpha, x = _problem(q, m, n, g, batch, seed=5)
        full = _oracle(x, signs, alpha, g)
        # Rows: each rank's rows, gathered.
        pr = T.plan_rows(m, n, q, g, world, rank)
        s, a = T.take_shard(pr, signs, alpha)
        y = T.gather_rows(pr, _oracle(x, s, a, g), None)
        res["rows"] = float((y - full).abs().max() / full.abs().max())
        # Rows, one batch column and equal ranges: the direct gather.
        m_eq = 64 * world
        s_eq, a_eq, x_eq = _problem(q, m_eq, n, g, 1, seed=8)
        pe = T.plan_rows(m_eq, n, q, g, world, rank)
        assert pe.m == pe.world * pe.span
        se, ae = T.take_shard(pe, s_eq, a_eq)
        ye = T.gather_rows(pe, _oracle(x_eq, se, ae, g), None)
        full_eq = _oracle(x_eq, s_eq, a_eq, g)
        res["rows_eq"] = float((ye - full_eq).abs().max() / full_eq.abs().max())
        # Inputs: each rank's partial product over its groups, summed.
        pi = T.plan_inputs(m, n, q, g, world, rank)
        s, a = T.take_shard(pi, signs, alpha)
        part = _oracle(T.take_input_slice(pi, x), s, a, g)
        y = T.reduce_inputs(pi, part.clone(), None)
        res["inputs"] = float((y - full).abs().max() / full.abs().max())
        # Inputs, summed and split by rows.
        rows, yr = T.reduce_scatter_inputs(pi, part.clone(), None)
        res["scatter"] = float((yr - full[:, rows.lo:rows.hi]).abs().max() / full.abs().max())
        res["scatter_rows"] = [rows.lo, rows.hi]
        # Paired block: W1 by rows -> fp16 hidden slice -> W2 by inputs, one all-reduce.
        m1, n1, m2 = 256, 256, 96
        s1, a1, x1 = _problem(q, m1, n1, g, batch, seed=6)
        s2, a2, _ = _problem(q, m2, m1, g, batch, seed=7)
        h = _oracle(x1, s1, a1, g).to(torch.float16)
        ref = _oracle(h, s2, a2, g)
        p1, p2 = T.plan_paired(m1, n1, m2, q, g, world, rank)
        ls1, la1 = T.take_shard(p1, s1, a1)
        ls2, la2 = T.take_shard(p2, s2, a2)
        h_local = _oracle(x1, ls1, la1, g).to(torch.float16)
        y = T.reduce_inputs(p2, _oracle(h_local, ls2, la2, g), None)
        res["paired"] = float((y - ref).abs().max() / ref.abs().max())
        import json
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_products_equal_the_whole_matrix(tmp_path, world):
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    import json
    seen_rows = []
    for r in range(world):
        res = json.load(open(tmp_path / f"rank{r}.json"))
        # FP64 on both sides: only the summation order differs.
        assert res["rows"] < 1e-13, res
        assert res["rows_eq"] < 1e-13, res
        assert res["inputs"] < 1e-13, res
        assert res["scatter"] < 1e-13, res
        assert res["paired"] < 1e-12, res
        seen_rows.append(tuple(res["scatter_rows"]))
    assert seen_rows[0][0] == 0 and seen_rows[-1][1] == 200
    assert all(a[1] == b[0] for a, b in zip(seen_rows, seen_rows[1:]))
