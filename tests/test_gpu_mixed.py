"""Mixed storage on the GPU (lutgemm_pack_bcq_mixed, lutgemm_run_mixed)
against the oracle's mixed format.

The format follows this library's reading of the OpenAlex record "Fast and
Efficient 2-bit LLM Inference on GPU: 2/4/16-bit in a Weight Matrix with
Asynchronous Dequantization" (abstract): 32-row x 1024-input blocks carry their
own number of planes, sparse fp16 outliers are added.  Packing is compared bit
for bit; the product within the matmul tolerance, with A_j taken over the
scales the blocks actually use.  Corrupted block tables and outlier entries are
caught by the kernel's own range checks and reported in the status word.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import bcq_synth as S
from oracle import bcq_oracle as O
from tests._guard import Guarded
from tests._tol import compare, compare_f16

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def L():
    from weight_only_quantized_bcq_b200 import lutgemm
    lutgemm.lib()
    assert torch.cuda.is_available()
    return lutgemm


def _problem(seed, q_max, m, n, g, batch, frac_hi, density, lo=2):
    gen = S.generator(seed)
    bp = S.draw_block_planes(gen, m, n, frac_hi, lo=min(lo, q_max), hi=q_max)
    signs = S.draw_signs(gen, q_max, m, n)
    alpha = S.draw_alpha(gen, q_max, m, n, g, 0.03)
    x = S.draw_x(gen, batch, n, outlier_frac=0.001)
    outl = S.draw_outliers(gen, m, n, density) if density > 0 else None
    return bp, signs, alpha, x, outl


def _effective_alpha(alpha, bp, m, n, g):
    """Scales with the planes a block does not store set to 0 (for A_j)."""
    a = alpha.numpy().astype(np.float64).copy()
    q = a.shape[0]
    for G in range(n // g):
        s_ = (G * g) // 1024
        for R in range(-(-m // 32)):
            qb = int(bp[s_, R])
            a[qb:, G, 32 * R: 32 * R + 32] = 0.0
    return a


def _device(L, bp, signs, outl, m, n):
    q_max = signs.shape[0]
    boff = L.mixed_offsets(bp, q_max, m, n).to(DEV)
    flags = torch.zeros(1, dtype=torch.int32, device=DEV)
    packed = L.pack_bcq_mixed(signs.to(DEV), boff, status_flags=flags)
    optr = oent = None
    if outl is not None:
        optr, oent = L.pack_outliers(*outl, m, n)
        optr, oent = optr.to(DEV), oent.to(DEV)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    return boff, packed, optr, oent


@pytest.mark.parametrize("q_max,m,n", [(4, 40, 2048), (4, 100, 3000), (2, 33, 1032), (3, 257, 5120), (1, 64, 1024)])
def test_pack_mixed_bit_exact(L, q_max, m, n):
    bp, signs, _, _, _ = _problem(q_max * 7 + m, q_max, m, n, 8, 1, 0.3, 0.0, lo=1)
    boff, packed, _, _ = _device(L, bp, signs, None, m, n)
    want = O.pack_mixed(signs.numpy(), bp.numpy())
    assert packed.numel() == want.size
    assert np.array_equal(packed.cpu().numpy(), want)


CASES = [
    # q_max, m, n, g, batch, frac_hi, density
    (4, 512, 2048, 64, 1, 0.25, 0.005),
    (4, 100, 3000, 40, 2, 0.5, 0.01),         # ragged rows and slice, g not a power of two
    (4, 257, 4096, 128, 3, 0.125, 0.0),        # no outliers
    (2, 300, 2048, 8, 1, 0.5, 0.02),           # one scale per run; 1- and 2-plane blocks
    (3, 64, 2048, 256, 4, 0.4, 0.003),
    (4, 2048, 4096, 64, 37, 0.125, 0.005),     # counter-taken tiles (148 segments)
    (4, 8192, 8192, 64, 1, 0.125, 0.005),      # LLaMA-70B q/k/v/o-shaped
]


@pytest.mark.parametrize("q_max,m,n,g,batch,frac_hi,density", CASES)
def test_run_mixed_matches_oracle(L, q_max, m, n, g, batch, frac_hi, density):
    bp, signs, alpha, x, outl = _problem(500 + q_max * 13 + m + batch, q_max, m, n, g, batch, frac_hi, density,
                                         lo=1 if q_max < 4 else 2)
    boff, packed, optr, oent = _device(L, bp, signs, outl, m, n)
    ws = Guarded(L.workspace_size(m, n, batch, q_max, g), torch.uint8, fill=0)
    y = Guarded(batch * m, torch.float32, shape=(batch, m))
    L.run_mixed(packed, boff, alpha.to(DEV), x.to(DEV), m, n, q_max, g, optr=optr, oent=oent, y=y.t,
                workspace=ws.t, check=True)
    torch.cuda.synchronize()
    assert ws.intact() and y.intact()
    got = y.t.cpu().numpy()
    assert np.all(np.isfinite(got)), "an output was never written"
    o = None if outl is None else tuple(t.numpy() for t in outl)
    y_ref = O.mixed_matmul(x.numpy(), signs.numpy(), alpha.numpy(), bp.numpy(), g, o)
    ok, st = compare(got, y_ref, _effective_alpha(alpha, bp.numpy(), m, n, g), x.numpy(), n)
    assert ok, st


def test_run_mixed_fp16_and_reruns(L):
    q_max, m, n, g, batch = 4, 700, 5120, 64, 2
    bp, signs, alpha, x, outl = _problem(77, q_max, m, n, g, batch, 0.2, 0.005)
    boff, packed, optr, oent = _device(L, bp, signs, outl, m, n)
    a_d, x_d = alpha.to(DEV), x.to(DEV)
    ws = L.new_workspace(m, n, batch, q_max, g)
    y32 = [L.run_mixed(packed, boff, a_d, x_d, m, n, q_max, g, optr=optr, oent=oent, workspace=ws).clone()
           for _ in range(3)]
    y16 = L.run_mixed(packed, boff, a_d, x_d, m, n, q_max, g, optr=optr, oent=oent, workspace=ws, y_f16=True)
    assert L.workspace_status(ws) == 0
    assert torch.equal(y32[0], y32[1]) and torch.equal(y32[0], y32[2])
    assert torch.equal(y16, y32[0].to(torch.float16))
    y_ref = O.mixed_matmul(x.numpy(), signs.numpy(), alpha.numpy(), bp.numpy(), g, tuple(t.numpy() for t in outl))
    ok, st = compare_f16(y16.cpu().numpy(), y_ref, _effective_alpha(alpha, bp.numpy(), m, n, g), x.numpy(), n)
    assert ok, st


def test_all_blocks_at_q_give_lutgemm_run_bits(L):
    """Every block at q = 2 planes and no outliers: the same bits as
    lutgemm_run on the uniform layout (the buffers are equal)."""
    q, m, n, g, batch = 2, 300, 3072, 64, 2
    gen = S.generator(31)
    signs = S.draw_signs(gen, q, m, n)
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02).to(DEV)
    x = S.draw_x(gen, batch, n).to(DEV)
    bp = torch.full((-(-n // 1024), -(-m // 32)), q, dtype=torch.uint8)
    boff, packed, _, _ = _device(L, bp, signs, None, m, n)
    assert torch.equal(packed, L.pack_bcq(signs.to(DEV)))
    y_mixed = L.run_mixed(packed, boff, alpha, x, m, n, q, g, check=True)
    y_run = L.run(packed, alpha, x, m, n, q, g, check=True)
    # Same tables, same ring, same plane order: the same terms in the same order.
    assert torch.equal(y_mixed, y_run)


def test_full_size_llama_up_sampled_tiles(L):
    """LLaMA-70B up-projection shape (28672 x 8192), 2/4-bit blocks and 0.5%
    outliers at batch 4: 48 row tiles (first and last included), every row
    of them, against the oracle on those rows."""
    q_max, m, n, g, batch = 4, 28672, 8192, 64, 4
    gen = S.generator(4040)
    bp = S.draw_block_planes(gen, m, n, 0.125)
    boff_h = L.mixed_offsets(bp, q_max, m, n)
    total = int(boff_h[-1])
    packed = S.draw_random_bytes(gen, total * 4096)
    alpha = S.draw_alpha(gen, q_max, m, n, g, 0.03)
    x = S.draw_x(gen, batch, n, outlier_frac=0.001)
    rp, col, val = S.draw_outliers(gen, m, n, 0.005)
    optr, oent = L.pack_outliers(rp, col, val, m, n)
    y = L.run_mixed(packed.to(DEV), boff_h.to(DEV), alpha.to(DEV), x.to(DEV), m, n, q_max, g,
                    optr=optr.to(DEV), oent=oent.to(DEV), check=True)
    mt = m // 32
    tiles = np.unique(np.r_[0, mt - 1, np.random.default_rng(5).choice(mt, 46, replace=False)])
    y_ref, rows = O.mixed_matmul_tiles(x.numpy(), packed.numpy(), bp.numpy(), alpha.numpy(), g, m, n, tiles,
                                       (rp.numpy(), col.numpy(), val.numpy()))
    a_eff = _effective_alpha(torch.from_numpy(alpha.numpy()[:, :, rows]), bp.numpy()[:, tiles], rows.size, n, g)
    ok, st = compare(y.cpu().numpy()[:, rows], y_ref, a_eff, x.numpy(), n)
    assert ok, st


def test_corrupt_block_table_is_reported_not_read(L):
    """A block-table entry with no plane, or one pointing past the buffer, is
    caught by the kernel's range check: LUTGEMM_STATUS_FORMAT, no access
    outside the buffers, and the next call with the good table is right."""
    q_max, m, n, g, batch = 4, 256, 4096, 64, 1
    bp, signs, alpha, x, outl = _problem(12, q_max, m, n, g, batch, 0.25, 0.005)
    boff, packed, optr, oent = _device(L, bp, signs, outl, m, n)
    a_d, x_d = alpha.to(DEV), x.to(DEV)
    ws = L.new_workspace(m, n, batch, q_max, g)
    for corrupt in ("empty", "past_end"):
        bad = boff.clone()
        if corrupt == "empty":
            bad[3] = bad[2]                                   # block 2 has no plane
        else:
            bad[-1] = bad[-1] + 4                              # last block ends past the buffer
        L.run_mixed(packed, bad, a_d, x_d, m, n, q_max, g, optr=optr, oent=oent, workspace=ws)
        assert L.workspace_status(ws) == L.STATUS_FORMAT
    y = L.run_mixed(packed, boff, a_d, x_d, m, n, q_max, g, optr=optr, oent=oent, workspace=ws, check=True)
    y_ref = O.mixed_matmul(x.numpy(), signs.numpy(), alpha.numpy(), bp.numpy(), g, tuple(t.numpy() for t in outl))
    ok, st = compare(y.cpu().numpy(), y_ref, _effective_alpha(alpha, bp.numpy(), m, n, g), x.numpy(), n)
    assert ok, st


def test_corrupt_outlier_entries_are_reported_not_read(L):
    q_max, m, n, g = 4, 128, 2048, 64
    bp, signs, alpha, x, outl = _problem(13, q_max, m, n, g, 1, 0.25, 0.01)
    boff, packed, optr, oent = _device(L, bp, signs, outl, m, n)
    ws = L.new_workspace(m, n, 1, q_max, g)
    bad = oent.clone()
    bad[0] = (bad[0] & ~0xFFFF) | 0x7FF                       # input 2047 of a slice: outside 1024
    L.run_mixed(packed, boff, alpha.to(DEV), x.to(DEV), m, n, q_max, g, optr=optr, oent=bad, workspace=ws)
    assert L.workspace_status(ws) == L.STATUS_FORMAT
    bad_ptr = optr.clone()
    bad_ptr[-1] = bad_ptr[-1] + 100                            # past the entries
    L.run_mixed(packed, boff, alpha.to(DEV), x.to(DEV), m, n, q_max, g, optr=bad_ptr, oent=oent, workspace=ws)
    assert L.workspace_status(ws) == L.STATUS_FORMAT


def test_mixed_stall_hook_reports_timeout(L):
    q_max, m, n, g = 4, 512, 2048, 64
    bp, signs, alpha, x, outl = _problem(14, q_max, m, n, g, 1, 0.25, 0.005)
    boff, packed, optr, oent = _device(L, bp, signs, outl, m, n)
    ws = L.new_workspace(m, n, 1, q_max, g)
    L.run_mixed(packed, boff, alpha.to(DEV), x.to(DEV), m, n, q_max, g, optr=optr, oent=oent, workspace=ws,
                _flags=L.TEST_STALL)
    assert L.workspace_status(ws) == L.STATUS_TIMEOUT


# ---------------------------------------------------------------------------
# Unit-major scales of mixed storage: bit-exact packing, and the product with
# them gives the bits of the product with [q_max][n/g][m] scales.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("q_max,m,n,g,lo", [(4, 100, 3072, 64, 1), (3, 70, 2048, 128, 1), (4, 64, 2048, 256, 2),
                                            (2, 33, 1152, 128, 1), (4, 40, 1024, 64, 3)])
def test_pack_scales_mixed_bit_exact(L, q_max, m, n, g, lo):
    gen = S.generator(600 + q_max * 7 + m)
    bp = S.draw_block_planes(gen, m, n, 0.4, lo=lo, hi=q_max)
    alpha = S.draw_alpha(gen, q_max, m, n, g, 0.03)
    boff = L.mixed_offsets(bp, q_max, m, n).to(DEV)
    flags = torch.zeros(1, dtype=torch.int32, device=DEV)
    sc = L.pack_scales_mixed(alpha.to(DEV), boff, m, n, g, status_flags=flags)
    torch.cuda.synchronize()
    want = O.pack_mixed_scales(alpha.numpy(), bp.numpy(), g)
    assert int(flags.item()) == 0
    assert sc.numel() == want.size
    assert np.array_equal(sc.cpu().numpy().view(np.uint16), want.view(np.uint16))


@pytest.mark.parametrize("q_max,m,n,g,batch,lo,density", [
    (4, 512, 2048, 64, 1, 2, 0.005),
    (3, 257, 4096, 128, 3, 1, 0.0),       # 1- and 3-plane blocks: one-plane passes
    (4, 2048, 4096, 64, 37, 1, 0.005),    # counter-taken tiles, every plane count
    (2, 300, 2048, 256, 2, 1, 0.01),
])
def test_run_mixed_packed_scales_same_bits(L, q_max, m, n, g, batch, lo, density):
    bp, signs, alpha, x, outl = _problem(700 + q_max + m, q_max, m, n, g, batch, 0.4, density, lo=lo)
    boff, packed, optr, oent = _device(L, bp, signs, outl, m, n)
    a_d, x_d = alpha.to(DEV), x.to(DEV)
    sc = L.pack_scales_mixed(a_d, boff, m, n, g)
    y_raw = L.run_mixed(packed, boff, a_d, x_d, m, n, q_max, g, optr=optr, oent=oent, check=True)
    y_pk = L.run_mixed(packed, boff, sc, x_d, m, n, q_max, g, optr=optr, oent=oent, scales_packed=True, check=True)
    assert torch.equal(y_raw, y_pk)
    o = None if outl is None else tuple(t.numpy() for t in outl)
    y_ref = O.mixed_matmul(x.numpy(), signs.numpy(), alpha.numpy(), bp.numpy(), g, o)
    ok, st = compare(y_pk.cpu().numpy(), y_ref, _effective_alpha(alpha, bp.numpy(), m, n, g), x.numpy(), n)
    assert ok, st


def test_full_size_llama_up_packed_scales(L):
    """The bench's configuration: LLaMA-70B up-projection, 2/4-plane blocks,
    0.5 % outliers, unit-major scales, batch 1; 48 row tiles against the oracle."""
    q_max, m, n, g = 4, 28672, 8192, 64
    gen = S.generator(4141)
    bp = S.draw_block_planes(gen, m, n, 0.125)
    boff_h = L.mixed_offsets(bp, q_max, m, n)
    packed = S.draw_random_bytes(gen, int(boff_h[-1]) * 4096)
    alpha = S.draw_alpha(gen, q_max, m, n, g, 0.03)
    x = S.draw_x(gen, 1, n, outlier_frac=0.001)
    rp, col, val = S.draw_outliers(gen, m, n, 0.005)
    optr, oent = L.pack_outliers(rp, col, val, m, n)
    boff = boff_h.to(DEV)
    sc = L.pack_scales_mixed(alpha.to(DEV), boff, m, n, g)
    y = L.run_mixed(packed.to(DEV), boff, sc, x.to(DEV), m, n, q_max, g, optr=optr.to(DEV), oent=oent.to(DEV),
                    scales_packed=True, check=True)
    mt = m // 32
    tiles = np.unique(np.r_[0, mt - 1, np.random.default_rng(6).choice(mt, 46, replace=False)])
    y_ref, rows = O.mixed_matmul_tiles(x.numpy(), packed.numpy(), bp.numpy(), alpha.numpy(), g, m, n, tiles,
                                       (rp.numpy(), col.numpy(), val.numpy()))
    a_eff = _effective_alpha(torch.from_numpy(alpha.numpy()[:, :, rows]), bp.numpy()[:, tiles], rows.size, n, g)
    ok, st = compare(y.cpu().numpy()[:, rows], y_ref, a_eff, x.numpy(), n)
    assert ok, st
