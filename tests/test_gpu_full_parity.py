"""Every output against the FP64 oracle on the paths the kernel takes at full size.

The lookup kernel hands row tiles out in two ways.  Small problems cut the
list of (batch column, slice, row tile) units into one contiguous range per
CTA.  Large ones give every (batch column, slice) segment its own group of
CTAs: each warp takes two row tiles, and the rest of the segment's tiles go to
whichever warp asks first, through a per-segment tile counter.  The cases here
are chosen (and checked, through lutgemm_launch_plan) to take the counter
path, and every output is compared with the oracle, so a tile that were
skipped or done twice would show.  Outputs start as NaN so an unwritten one
cannot pass; every output buffer sits between guard bytes that must survive.

The oracle's result (dequantise, then matmul, in FP64) is what the lookup
form must reproduce: the LUT-GEMM card (Summary) says the product needs no
dequantisation, which is an exact regrouping of that sum.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import bcq_synth as S
from oracle import bcq_oracle as O
from tests._guard import Guarded
from tests._oracle_pool import oracle_all_rows
from tests._tol import compare, compare_f16

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def L():
    from weight_only_quantized_bcq_b200 import lutgemm
    lutgemm.lib()
    assert torch.cuda.is_available()
    return lutgemm


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _dyn_plan(L, m, n, batch):
    grid, aligned, dyn = L.launch_plan(m, n, batch, _sms())
    assert aligned == 1 and dyn > 0, (m, n, batch, grid, aligned, dyn)
    return dyn


DYN_CASES = [
    # q, m, n, g, batch, offsets, y_f16
    (3, 2048, 4096, 128, 37, False, False),    # 148 segments of one CTA: 32 of 64 tiles by counter
    (2, 12600, 12288, 64, 1, False, False),    # ragged last tile (24 rows), g = 64
    (3, 2048, 4096, 128, 37, True, False),     # offsets (converted uniform weights)
    (5, 2048, 4096, 256, 37, False, False),    # q > 4: two plane groups per unit
    (3, 2080, 4096, 8, 37, False, True),       # one scale per run, fp16 y
    (4, 6000, 5000, 40, 6, False, False),      # 30 segments, ragged last slice, g = 40
]


@pytest.mark.parametrize("q,m,n,g,batch,with_off,y_f16", DYN_CASES)
def test_dynamic_tiles_every_output(L, q, m, n, g, batch, with_off, y_f16):
    dyn = _dyn_plan(L, m, n, batch)
    gen = S.generator(9000 + q * 31 + m)
    signs = S.draw_signs(gen, q, m, n)
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02)
    x = S.draw_x(gen, batch, n)
    off = (torch.randn((n // g, m), generator=gen) * 0.05).float() if with_off else None
    pk = Guarded(L.packed_bytes(q, m, n), torch.uint8, fill=0)
    L.pack_bcq(signs.to(DEV), packed=pk.t)
    ws = Guarded(L.workspace_size(m, n, batch, q, g), torch.uint8, fill=0)
    y = Guarded(batch * m, torch.float16 if y_f16 else torch.float32, shape=(batch, m))
    L.run(pk.t, alpha.to(DEV), x.to(DEV), m, n, q, g, offset=None if off is None else off.to(DEV),
          y=y.t, workspace=ws.t, y_f16=y_f16, check=True)
    torch.cuda.synchronize()
    assert pk.intact() and ws.intact() and y.intact()
    got = y.t.float().cpu().numpy()
    assert np.all(np.isfinite(got)), "an output was never written"
    y_ref = O.bcq_matmul(x.numpy(), signs.numpy(), alpha.numpy(), g, None if off is None else off.numpy())
    if y_f16:
        # The fp16 mode rounds the fp32 sum to nearest even: the same call with
        # fp32 y meets the matmul tolerance, and its rounding is y bit for bit.
        y32 = L.run(pk.t, alpha.to(DEV), x.to(DEV), m, n, q, g, offset=None if off is None else off.to(DEV),
                    check=True)
        ok, st = compare(y32.cpu().numpy(), y_ref, alpha.numpy(), x.numpy(), n)
        assert ok, (st, dyn)
        assert torch.equal(y.t, y32.to(torch.float16))
        ok16, st16 = compare_f16(y.t.cpu().numpy(), y_ref, alpha.numpy(), x.numpy(), n)
        assert ok16, st16
    else:
        ok, st = compare(got, y_ref, alpha.numpy(), x.numpy(), n)
        assert ok, (st, dyn)
    # Tile counters are zero again after the call.
    assert not ws.t[256: 256 + 4096].cpu().numpy().any()


def test_dynamic_tiles_reruns_are_bit_identical(L):
    """Which warp takes which counter tile varies from run to run; the sums
    of a tile do not depend on it."""
    q, m, n, g, batch = 3, 2048, 4096, 128, 37
    _dyn_plan(L, m, n, batch)
    gen = S.generator(4242)
    packed = S.draw_random_bytes(gen, L.packed_bytes(q, m, n)).to(DEV)
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02).to(DEV)
    x = S.draw_x(gen, batch, n).to(DEV)
    ws = L.new_workspace(m, n, batch, q, g)
    ys = [L.run(packed, alpha, x, m, n, q, g, workspace=ws).clone() for _ in range(5)]
    torch.cuda.synchronize()
    assert L.workspace_status(ws) == 0
    for y in ys[1:]:
        assert torch.equal(y, ys[0])


def test_fc1_every_row_as_the_bench_runs_it(L):
    """OPT-175B FC1 (49152 x 12288, q = 3, g = 128, batch 1) with unit-major
    scales, the bench's configuration: 1152 of each segment's 1536 row tiles
    go through the counters.  All 49152 outputs against the oracle."""
    m, n, q, g = 49152, 12288, 3, 128
    _dyn_plan(L, m, n, 1)
    gen = S.generator(2)
    packed = S.draw_random_bytes(gen, O.packed_nbytes(q, m, n))
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02)
    x = S.draw_x(gen, 1, n)
    scales = L.pack_scales(alpha.to(DEV), m, n, g)
    y = Guarded(m, torch.float32, shape=(1, m))
    L.run(packed.to(DEV), scales, x.to(DEV), m, n, q, g, y=y.t, scales_packed=True, check=True)
    torch.cuda.synchronize()
    assert y.intact()
    got = y.t.cpu().numpy()
    y_ref = oracle_all_rows(packed.numpy(), q, m, n, alpha.numpy(), x.numpy(), g)
    ok, st = compare(got, y_ref, alpha.numpy(), x.numpy(), n)
    assert ok, st


# ---------------------------------------------------------------------------
# Guard bytes around every output of the other paths: ragged m, fp16 y, split
# K, the conversion outputs, the unit-major scales, the tensor cores with and
# without K splits.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("q,m,n,g,batch,y_f16", [(3, 45, 2056, 8, 2, False), (2, 70, 3000, 40, 3, True),
                                                 (1, 1, 8, 8, 1, False), (8, 33, 1032, 8, 1, True)])
def test_guards_lookup_path(L, q, m, n, g, batch, y_f16):
    gen = S.generator(77 + q + m)
    signs = S.draw_signs(gen, q, m, n)
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02)
    x = S.draw_x(gen, batch, n)
    pk = Guarded(L.packed_bytes(q, m, n), torch.uint8, fill=0x5A)
    L.pack_bcq(signs.to(DEV), packed=pk.t)
    ws = Guarded(L.workspace_size(m, n, batch, q, g), torch.uint8, fill=0)
    y = Guarded(batch * m, torch.float16 if y_f16 else torch.float32, shape=(batch, m))
    L.run(pk.t, alpha.to(DEV), x.to(DEV), m, n, q, g, y=y.t, workspace=ws.t, y_f16=y_f16, check=True)
    torch.cuda.synchronize()
    assert pk.intact() and ws.intact() and y.intact()
    assert np.array_equal(pk.t.cpu().numpy(), O.pack_bcq(signs.numpy()))
    got = y.t.float().cpu().numpy()
    assert np.all(np.isfinite(got))
    if not y_f16:
        ok, st = compare(got, O.bcq_matmul(x.numpy(), signs.numpy(), alpha.numpy(), g), alpha.numpy(),
                         x.numpy(), n)
        assert ok, st


def test_guards_uniform_conversion_and_scales(L):
    q, m, n, g = 4, 97, 2048, 128
    codes, scale, zero = S.draw_uniform(S.generator(5), m, n, g, q, 0.01)
    dev_codes, dev_scale, dev_zero = codes.to(DEV), scale.to(DEV), zero.to(DEV)
    lib = L.lib()
    import ctypes
    pk = Guarded(L.packed_bytes(q, m, n), torch.uint8, fill=0x5A)
    al = Guarded(q * (n // g) * m, torch.float16)
    of = Guarded((n // g) * m, torch.float32)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib.lutgemm_uniform_to_bcq(ptr(dev_codes), ptr(dev_scale), ptr(dev_zero), q, m, n, g, ptr(pk.t),
                                    ptr(al.t), ptr(of.t), None,
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == L.OK
    sc = Guarded(L.scales_bytes(q, m, n, g) // 2, torch.float16)
    st = lib.lutgemm_pack_scales(ptr(al.t), q, m, n, g, ptr(sc.t),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == L.OK
    torch.cuda.synchronize()
    assert pk.intact() and al.intact() and of.intact() and sc.intact()
    s_ref, a_ref, o_ref = O.uniform_to_bcq(codes.numpy(), scale.numpy(), zero.numpy(), q, g)
    assert np.array_equal(pk.t.cpu().numpy(), O.pack_bcq(s_ref))
    assert np.array_equal(al.t.cpu().numpy().view(np.uint16), a_ref.reshape(-1).view(np.uint16))
    assert np.array_equal(of.t.cpu().numpy().view(np.uint32), o_ref.reshape(-1).view(np.uint32))
    assert np.array_equal(sc.t.cpu().numpy().view(np.uint16), O.pack_scales(a_ref, g).view(np.uint16))


@pytest.mark.parametrize("m,n,batch,allow", [(300, 4096, 40, False), (12288, 12288, 64, True)])
def test_guards_tensor_core_paths(L, m, n, batch, allow):
    """lutgemm_run_tc (one split) and lutgemm_run's tensor-core dispatch, which
    splits K for short, long matrices (partials in the workspace)."""
    q, g = 3, 128
    gen = S.generator(m + batch)
    packed = S.draw_random_bytes(gen, O.packed_nbytes(q, m, n))
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02)
    x = S.draw_x(gen, batch, n)
    y = Guarded(batch * m, torch.float32, shape=(batch, m))
    if allow:
        assert L.tc_plan(m, n, batch, q, _sms()) > 1        # the split-K form
        ws = Guarded(L.workspace_size(m, n, batch, q, g), torch.uint8, fill=0)
        L.run(packed.to(DEV), alpha.to(DEV), x.to(DEV), m, n, q, g, y=y.t, workspace=ws.t,
              allow_tensor_cores=True, check=True)
    else:
        ws = None
        L.run_tc(packed.to(DEV), alpha.to(DEV), x.to(DEV), m, n, q, g, y=y.t, check=True)
    torch.cuda.synchronize()
    assert y.intact() and (ws is None or ws.intact())
    got = y.t.cpu().numpy()
    assert np.all(np.isfinite(got))
    rows = np.unique(np.r_[0, 31, 32, m // 2, m - 33, m - 1, np.random.default_rng(1).integers(0, m, 40)])
    s_rows = O.unpack_rows(packed.numpy(), q, m, n, rows)
    a_rows = alpha.numpy()[:, :, rows]
    ok, st = compare(got[:, rows], O.bcq_matmul_rows(x.numpy(), s_rows, a_rows, g), a_rows, x.numpy(), n)
    assert ok, st
