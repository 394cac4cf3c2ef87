"""Tensor-parallel LUT-GEMM on the GPU.

This pool gives one GPU per run, so the multi-rank exchange itself is covered
on the CPU (tests/test_sharded_cpu.py, gloo).  Here:

* every shard of a 2- and 3-way split runs through the CUDA library on one
  GPU, in one process (no rank waits on another); row shards must give the
  whole product's rows bit for bit, input shards must sum to it within the
  matmul tolerance;
* ShardedLinear and paired_block run end to end over a one-rank NCCL group.
"""
from __future__ import annotations

import datetime
import socket

import numpy as np
import pytest
import torch

import bcq_synth as S
from oracle import bcq_oracle as O
from tests._tol import compare

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def L():
    from weight_only_quantized_bcq_b200 import lutgemm
    lutgemm.lib()
    assert torch.cuda.is_available()
    return lutgemm


@pytest.fixture(scope="module")
def T():
    from weight_only_quantized_bcq_b200 import sharded
    return sharded


@pytest.fixture(scope="module")
def nccl_group():
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    yield dist.group.WORLD
    dist.destroy_process_group()


def _problem(seed, q, m, n, g, batch):
    gen = S.generator(seed)
    return S.draw_signs(gen, q, m, n), S.draw_alpha(gen, q, m, n, g, 0.02), S.draw_x(gen, batch, n)


def _run(L, signs, alpha, x, q, g):
    _, m, n = signs.shape
    return L.run(L.pack_bcq(signs.to(DEV)), alpha.to(DEV), x.to(DEV), m, n, q, g)


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("q,m,n,g,batch", [(3, 1000, 3072, 128, 1), (2, 300, 2560, 64, 4)])
def test_every_shard_on_the_gpu_recombines_to_the_whole(L, T, world, q, m, n, g, batch):
    signs, alpha, x = _problem(70 + world, q, m, n, g, batch)
    full = _run(L, signs, alpha, x, q, g).cpu()
    ref = O.bcq_matmul(x.numpy(), signs.numpy(), alpha.numpy(), g)
    rows = []
    part_sum = torch.zeros_like(full, dtype=torch.float64)
    for r in range(world):
        pr = T.plan_rows(m, n, q, g, world, r)
        s, a = T.take_shard(pr, signs, alpha)
        rows.append(_run(L, s, a, x, q, g).cpu())
        pi = T.plan_inputs(m, n, q, g, world, r)
        s, a = T.take_shard(pi, signs, alpha)
        part_sum += _run(L, s, a, T.take_input_slice(pi, x), q, g).cpu().double()
    # A row's arithmetic does not depend on the other rows: bit for bit.
    assert torch.equal(torch.cat(rows, 1), full)
    # Input shards change the summation order only.
    ok, st = compare(part_sum.numpy(), ref, alpha.numpy(), x.numpy(), n)
    assert ok, st


def test_sharded_linear_over_nccl(L, T, nccl_group):
    q, m, n, g, batch = 3, 640, 2048, 128, 3
    signs, alpha, x = _problem(81, q, m, n, g, batch)
    full = _run(L, signs, alpha, x, q, g)
    pr = T.plan_rows(m, n, q, g, 1, 0)
    s, a = T.take_shard(pr, signs.to(DEV), alpha.to(DEV))
    lin = T.ShardedLinear(pr, s, a, group=nccl_group, batch=batch)
    assert torch.equal(lin(x.to(DEV)), full)
    pi = T.plan_inputs(m, n, q, g, 1, 0)
    s, a = T.take_shard(pi, signs.to(DEV), alpha.to(DEV))
    lin = T.ShardedLinear(pi, s, a, group=nccl_group, batch=batch)
    assert torch.equal(lin(x.to(DEV)), full)
    rows, yr = T.reduce_scatter_inputs(pi, full.clone(), nccl_group)
    assert (rows.lo, rows.hi) == (0, m) and torch.equal(yr, full)


def test_paired_block_over_nccl(L, T, nccl_group):
    q, g, batch = 3, 128, 2
    m1, n1, m2 = 1024, 512, 384
    s1, a1, x = _problem(91, q, m1, n1, g, batch)
    s2, a2, _ = _problem(92, q, m2, m1, g, batch)
    p1, p2 = T.plan_paired(m1, n1, m2, q, g, 1, 0)
    w1 = T.ShardedLinear(p1, *T.take_shard(p1, s1.to(DEV), a1.to(DEV)), group=nccl_group, batch=batch)
    w2 = T.ShardedLinear(p2, *T.take_shard(p2, s2.to(DEV), a2.to(DEV)), group=nccl_group, batch=batch)
    y = T.paired_block(w1, w2, x.to(DEV))
    h = _run(L, s1, a1, x, q, g).to(torch.float16)
    assert torch.equal(y, _run(L, s2, a2, h, q, g))
    ref = O.bcq_matmul(h.cpu().numpy(), s2.numpy(), a2.numpy(), g)
    ok, st = compare(y.cpu().numpy(), ref, a2.numpy(), h.cpu().numpy(), m1)
    assert ok, st
