"""GPU parity of BCQ fitting (lutgemm_fit_bcq) against the FP64 oracle.

The fit decides integers (signs) from floating-point comparisons, and the
kernel works in fp32 while the oracle works in fp64, so a handful of groups
may settle in a different local optimum.  What is unique is checked exactly
(closed forms, exact recovery, signs optimal for the stored scales, the
returned error); the rest is checked against the oracle statistically.
"""
from __future__ import annotations

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


def _check_signs_optimal(w, signs, alpha, g):
    """Each stored sign combination is a nearest one for the stored scales
    (fp64 check; a 2e-6 relative slack covers the kernel's fp32 comparisons)."""
    q, m, n = signs.shape
    W = w.astype(np.float64).reshape(m, n // g, g)
    A = alpha.astype(np.float64).transpose(2, 1, 0)                      # [m][ng][q]
    B = signs.astype(np.float64).reshape(q, m, n // g, g)
    v = np.einsum("mgq,qmgk->mgk", A, B)
    S_ = O._code_signs(q)                                                # [C][q]
    vals = np.einsum("cq,mgq->mgc", S_, A)
    best = np.abs(W[..., None] - vals[..., None, :]).min(-1)
    slack = 2e-6 * (np.abs(W) + np.abs(A).sum(-1, keepdims=True))
    assert np.all(np.abs(W - v) <= best + slack)
    return ((W - v) ** 2).sum(-1).T                                      # [ng][m]


def test_fit_q1_closed_form(L):
    w = S.draw_weights(S.generator(500), 64, 1024, 0.02)
    w[0, :7] = 0
    signs, alpha = L.fit_bcq(w.to(DEV), 1, 128, iters=3)
    torch.cuda.synchronize()
    wn = w.numpy().astype(np.float64)
    assert np.array_equal(signs.cpu().numpy()[0], np.where(wn >= 0, 1, -1))
    want = np.abs(wn).reshape(64, 8, 128).mean(-1).T.astype(np.float16)
    got = alpha.cpu().numpy()[0]
    ulp = np.spacing(np.abs(want)).astype(np.float64)
    assert np.all(np.abs(got.astype(np.float64) - want.astype(np.float64)) <= ulp)


def test_fit_recovers_representable_weights_exactly(L):
    rng = np.random.default_rng(501)
    m, ng, g = 48, 6, 128
    c = 2.0 ** rng.integers(-9, -4, size=(m, ng))
    b = rng.choice([-1.0, 1.0], size=(3, m, ng, g))
    w = (c[..., None] * (b[0] + b[1] / 2 + b[2] / 4)).reshape(m, ng * g).astype(np.float16)
    signs, alpha, err = L.fit_bcq(torch.from_numpy(w).to(DEV), 3, g, iters=3, with_error=True)
    torch.cuda.synchronize()
    assert np.array_equal(signs.cpu().numpy().reshape(3, m, ng, g), b.astype(np.int8))
    assert np.array_equal(alpha.cpu().numpy().astype(np.float64), np.stack([c, c / 2, c / 4]).transpose(0, 2, 1))
    assert float(err.abs().max()) == 0.0


@pytest.mark.parametrize("q,g,iters,m,n", [(2, 64, 3, 96, 2048), (3, 128, 0, 80, 3072), (3, 128, 3, 80, 3072),
                                           (4, 256, 2, 40, 4096), (8, 128, 2, 24, 1024), (3, 1024, 2, 16, 4096),
                                           (3, 8, 1, 32, 512)])
def test_fit_matches_oracle(L, q, g, iters, m, n):
    w = S.draw_weights(S.generator(600 + q * 10 + g), m, n, 0.02)
    signs, alpha, err = L.fit_bcq(w.to(DEV), q, g, iters=iters, with_error=True)
    torch.cuda.synchronize()
    s_np, a_np, e_np = signs.cpu().numpy(), alpha.cpu().numpy(), err.cpu().numpy().astype(np.float64)
    assert set(np.unique(s_np)) <= {-1, 1}
    e_exact = _check_signs_optimal(w.numpy(), s_np, a_np, g)
    assert np.allclose(e_np, e_exact, rtol=1e-4, atol=1e-12)
    o_signs, o_alpha, o_err = O.fit_bcq(w.numpy(), q, g, iters)
    # Same local optimum almost everywhere, same total error.
    same = np.all(s_np.reshape(q, m, n // g, g) == o_signs.reshape(q, m, n // g, g), axis=(0, 3)).T
    assert same.mean() >= 0.97, same.mean()
    assert abs(e_exact.sum() - o_err.sum()) <= 2e-3 * o_err.sum()
    ulp = np.spacing(np.abs(o_alpha).astype(np.float16)).astype(np.float64)
    close = np.abs(a_np.astype(np.float64) - o_alpha.astype(np.float64)) <= 2 * ulp
    assert close[:, same].all()


def test_fit_error_falls_with_rounds(L):
    w = S.draw_weights(S.generator(700), 128, 2048, 0.02)
    wd = w.to(DEV)
    _, _, e0 = L.fit_bcq(wd, 3, 128, iters=0, with_error=True)
    _, _, e3 = L.fit_bcq(wd, 3, 128, iters=3, with_error=True)
    torch.cuda.synchronize()
    e0, e3 = e0.cpu().numpy(), e3.cpu().numpy()
    scale = (w.numpy().astype(np.float64).reshape(128, 16, 128) ** 2).sum(-1).T
    # fp16 rounding of the scales can cost a little in a group; never more than it gains overall
    assert np.all(e3 <= e0 + 1e-3 * scale)
    assert e3.sum() < 0.95 * e0.sum()


def test_fit_is_deterministic(L):
    w = S.draw_weights(S.generator(701), 64, 4096, 0.02).to(DEV)
    a = L.fit_bcq(w, 4, 128, iters=3)
    b = L.fit_bcq(w, 4, 128, iters=3)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_fit_then_lutgemm_matches_oracle_product(L):
    """Fit -> pack -> run: y equals the oracle's product of the fitted BCQ weight."""
    m, n, q, g = 300, 3072, 3, 128
    gen = S.generator(702)
    w = S.draw_weights(gen, m, n, 0.02)
    x = S.draw_x(gen, 2, n)
    signs, alpha = L.fit_bcq(w.to(DEV), q, g, iters=3)
    packed = L.pack_bcq(signs)
    y = L.run(packed, alpha, x.to(DEV), m, n, q, g)
    torch.cuda.synchronize()
    y_ref = O.bcq_matmul(x.numpy(), signs.cpu().numpy(), alpha.cpu().numpy(), g)
    ok, st = compare(y.cpu().numpy(), y_ref, alpha.cpu().numpy(), x.numpy(), n)
    assert ok, st


def test_fit_full_size_sampled_rows(L):
    """OPT-175B FC1 shape (49152 x 12288), q = 3, g = 128, 3 rounds: sampled rows
    against the oracle fitting only those rows (rows are independent)."""
    m, n, q, g = 49152, 12288, 3, 128
    w = S.draw_weights(S.generator(703), m, n, 0.02)
    signs, alpha, err = L.fit_bcq(w.to(DEV), q, g, iters=3, with_error=True)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(703).choice(m, 24, replace=False))
    wr = w.numpy()[rows]
    o_signs, o_alpha, o_err = O.fit_bcq(wr, q, g, 3)
    s_np = signs[:, torch.from_numpy(rows)].cpu().numpy()
    a_np = alpha[:, :, torch.from_numpy(rows)].cpu().numpy()
    e_exact = _check_signs_optimal(wr, s_np, a_np, g)
    assert np.allclose(err[:, torch.from_numpy(rows)].cpu().numpy(), e_exact, rtol=1e-4, atol=1e-12)
    assert abs(e_exact.sum() - o_err.sum()) <= 2e-3 * o_err.sum()


# ---------------------------------------------------------------------------
# Variable grid (lutgemm_fit_bcq_grid): planes plus one constant per group.
# ---------------------------------------------------------------------------
def _shifted_weights(seed, m, n, sigma=0.02):
    """N(0, sigma) weights plus a per-row shift (what a constant per group can absorb)."""
    gen = S.generator(seed)
    w = S.draw_weights(gen, m, n, sigma).to(torch.float32)
    shift = torch.randn((m, 1), generator=gen) * sigma
    return (w + shift).to(torch.float16)


def _check_grid_points_nearest(w, signs, alpha, offset, g):
    q, m, n = signs.shape
    W = w.astype(np.float64).reshape(m, n // g, g)
    A = alpha.astype(np.float64).transpose(2, 1, 0)                      # [m][ng][q]
    off = offset.astype(np.float64).T                                    # [m][ng]
    B = signs.astype(np.float64).reshape(q, m, n // g, g)
    v = off[..., None] + np.einsum("mgq,qmgk->mgk", A, B)
    vals = off[..., None] + np.einsum("cq,mgq->mgc", O._code_signs(q), A)
    best = np.abs(W[..., None] - vals[..., None, :]).min(-1)
    slack = 2e-6 * (np.abs(W) + np.abs(off)[..., None] + np.abs(A).sum(-1, keepdims=True))
    assert np.all(np.abs(W - v) <= best + slack)
    return ((W - v) ** 2).sum(-1).T


def test_grid_recovers_representable_grids_exactly(L):
    rng = np.random.default_rng(520)
    m, ng, g = 40, 5, 128
    c = 2.0 ** rng.integers(-9, -5, size=(m, ng))
    off = rng.integers(-64, 64, size=(m, ng)) * 2.0 ** -12
    b = rng.choice([-1.0, 1.0], size=(2, m, ng, g))
    w = (off[..., None] + c[..., None] * (b[0] + b[1] / 2)).reshape(m, ng * g).astype(np.float16)
    signs, alpha, offset, err = L.fit_bcq_grid(torch.from_numpy(w).to(DEV), 2, g, iters=3, with_error=True)
    torch.cuda.synchronize()
    assert np.array_equal(signs.cpu().numpy().reshape(2, m, ng, g), b.astype(np.int8))
    assert np.array_equal(alpha.cpu().numpy().astype(np.float64), np.stack([c, c / 2]).transpose(0, 2, 1))
    # The constant comes out of an fp32 solve: exact up to fp32 rounding of the
    # group's magnitude (the FP64 oracle recovers it exactly).
    tol = 8 * np.spacing((np.abs(off) + 1.5 * c).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(offset.cpu().numpy().astype(np.float64) - off.T) <= tol.T)
    assert np.all(err.cpu().numpy() <= g * (tol.T ** 2))


@pytest.mark.parametrize("q,g,iters,m,n", [(1, 64, 3, 64, 1024), (2, 64, 3, 96, 2048), (3, 128, 3, 80, 3072),
                                           (4, 128, 2, 40, 2048), (6, 256, 2, 16, 1024)])
def test_grid_matches_oracle(L, q, g, iters, m, n):
    w = _shifted_weights(620 + q * 10 + g, m, n)
    signs, alpha, offset, err = L.fit_bcq_grid(w.to(DEV), q, g, iters=iters, with_error=True)
    torch.cuda.synchronize()
    s_np, a_np, o_np = signs.cpu().numpy(), alpha.cpu().numpy(), offset.cpu().numpy()
    e_exact = _check_grid_points_nearest(w.numpy(), s_np, a_np, o_np, g)
    assert np.allclose(err.cpu().numpy().astype(np.float64), e_exact, rtol=1e-4, atol=1e-12)
    o_signs, o_alpha, o_off, o_err = O.fit_bcq_grid(w.numpy(), q, g, iters)
    same = np.all(s_np.reshape(q, m, n // g, g) == o_signs.reshape(q, m, n // g, g), axis=(0, 3)).T
    assert same.mean() >= 0.97, same.mean()
    assert abs(e_exact.sum() - o_err.sum()) <= 2e-3 * o_err.sum()
    ulp = np.spacing(np.abs(o_alpha).astype(np.float16)).astype(np.float64)
    assert (np.abs(a_np.astype(np.float64) - o_alpha.astype(np.float64)) <= 2 * ulp)[:, same].all()
    # The constant comes out of the same fp32 solve: within fp32 rounding of the group's scale.
    tol = 1e-5 * (np.abs(o_off) + np.abs(o_alpha.astype(np.float64)).sum(0))
    assert (np.abs(o_np.astype(np.float64) - o_off.astype(np.float64)) <= tol)[same].all()
    # On shifted weights the grid beats the plain (zero-centred) BCQ fit.
    _, _, e_plain = L.fit_bcq(w.to(DEV), q, g, iters=iters, with_error=True)
    assert e_exact.sum() < e_plain.cpu().numpy().sum()


def test_grid_then_lutgemm_with_offset_matches_oracle_product(L):
    """Fit a grid -> pack -> lutgemm_run with the offset: the lookup kernel
    consumes the variable-grid format unchanged."""
    m, n, q, g = 260, 2048, 3, 128
    w = _shifted_weights(720, m, n)
    x = S.draw_x(S.generator(721), 3, n)
    signs, alpha, offset = L.fit_bcq_grid(w.to(DEV), q, g, iters=3)
    y = L.run(L.pack_bcq(signs), alpha, x.to(DEV), m, n, q, g, offset=offset)
    torch.cuda.synchronize()
    y_ref = O.bcq_matmul(x.numpy(), signs.cpu().numpy(), alpha.cpu().numpy(), g, offset.cpu().numpy())
    ok, st = compare(y.cpu().numpy(), y_ref, alpha.cpu().numpy(), x.numpy(), n)
    assert ok, st


def test_grid_is_deterministic(L):
    w = _shifted_weights(722, 64, 2048).to(DEV)
    a = L.fit_bcq_grid(w, 3, 128, iters=3)
    b = L.fit_bcq_grid(w, 3, 128, iters=3)
    torch.cuda.synchronize()
    assert all(torch.equal(u, v) for u, v in zip(a, b))
