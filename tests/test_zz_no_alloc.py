"""lutgemm_run_noalloc against lutgemm_run.

Some callers cannot allocate device memory (a runtime whose pool owns all of
it, a plugin host that hands over only input and output tensors), so they
cannot give lutgemm_run its workspace.  lutgemm_run_noalloc serves them from a
fixed scratch array inside the library.  These tests call it through the C ABI
and check that it gives what lutgemm_run gives, call after call, including
after a call of another shape has reused the same scratch.  The file is named
to be collected last.
"""
from __future__ import annotations

import ctypes
import math

import numpy as np
import pytest
import torch

import bcq_synth as S
from tests._tol import compare

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def L():
    from weight_only_quantized_bcq_b200 import lutgemm
    lutgemm.lib()
    assert torch.cuda.is_available()
    return lutgemm


def _inputs(seed, q, m, n, g, batch, with_off):
    gen = S.generator(seed)
    signs = S.draw_signs(gen, q, m, n)
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02)
    x = S.draw_x(gen, batch, n)
    off = (torch.randn((n // g, m), generator=gen) * 0.05).float() if with_off else None
    return signs, alpha, x, off


def _noalloc(L, packed, alpha, x, m, n, q, g, off=None):
    """One lutgemm_run_noalloc call through ctypes; y is the only buffer made here."""
    batch = x.shape[0]
    y = torch.empty((batch, m), dtype=torch.float32, device=DEV)
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = L.lib().lutgemm_run_noalloc(m, n, batch, q, g, ptr(packed), ptr(alpha), ptr(off), ptr(x), ptr(y), 0,
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == L.OK, L.status_string(st)
    return y


@pytest.mark.parametrize("q,m,n,g,batch,with_off", [
    (3, 1000, 6144, 128, 2, False),
    (2, 257, 3072, 64, 1, True),
    (4, 96, 5120, 128, 3, False),
])
def test_noalloc_matches_run_on_consecutive_calls(L, q, m, n, g, batch, with_off):
    signs, alpha, x, off = _inputs(q * 100 + m, q, m, n, g, batch, with_off)
    packed = L.pack_bcq(signs.to(DEV))
    a_d, x_d = alpha.to(DEV), x.to(DEV)
    o_d = None if off is None else off.to(DEV)
    y_run = L.run(packed, a_d, x_d, m, n, q, g, offset=o_d).cpu().numpy()
    for _ in range(2):
        y = _noalloc(L, packed, a_d, x_d, m, n, q, g, o_d)
        torch.cuda.synchronize()
        ok, st = compare(y.cpu().numpy(), y_run, alpha.numpy(), x.numpy(), n)
        assert ok, st


def test_noalloc_with_packed_scales_matches_run(L):
    """Unit-major scales through the no-alloc call give the bits of lutgemm_run."""
    q, m, n, g, batch = 3, 300, 3072, 128, 2
    signs, alpha, x, _ = _inputs(555, q, m, n, g, batch, False)
    packed = L.pack_bcq(signs.to(DEV))
    scales = L.pack_scales(alpha.to(DEV), m, n, g)
    x_d = x.to(DEV)
    y_run = L.run(packed, scales, x_d, m, n, q, g, scales_packed=True)
    y = L.run_noalloc(packed, scales, x_d, m, n, q, g, scales_packed=True)
    torch.cuda.synchronize()
    assert torch.equal(y, y_run)


def test_noalloc_full_size_layer_linear_twice(L):
    """The OPT-175B FC1 shape at batch 1 fits the scratch; two calls in a row."""
    m, n, q, g = 49152, 12288, 3, 128
    gen = S.generator(11)
    packed = S.draw_random_bytes(gen, L.packed_bytes(q, m, n)).to(DEV)
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02)
    x = S.draw_x(gen, 1, n)
    a_d, x_d = alpha.to(DEV), x.to(DEV)
    y_run = L.run(packed, a_d, x_d, m, n, q, g).cpu().numpy()
    for _ in range(2):
        y = _noalloc(L, packed, a_d, x_d, m, n, q, g)
        torch.cuda.synchronize()
        ok, st = compare(y.cpu().numpy(), y_run, alpha.numpy(), x.numpy(), n)
        assert ok, st


@pytest.mark.parametrize("y_f16", [False, True])
def test_noalloc_fp16_output_and_flags_match_run(L, y_f16):
    """With fp16 y, lutgemm_run_noalloc gives lutgemm_run's bits."""
    q, m, n, g, batch = 3, 700, 5120, 128, 2
    signs, alpha, x, _ = _inputs(808, q, m, n, g, batch, False)
    packed = L.pack_bcq(signs.to(DEV))
    a_d, x_d = alpha.to(DEV), x.to(DEV)
    y_run = L.run(packed, a_d, x_d, m, n, q, g, y_f16=y_f16)
    for _ in range(2):
        y = L.run_noalloc(packed, a_d, x_d, m, n, q, g, y_f16=y_f16, check=True)
        assert torch.equal(y, y_run)


def test_noalloc_tensor_cores_match_the_one_split_path(L):
    """With the tensor cores allowed and a plan of one K split (16384 x 12288,
    batch 16), lutgemm_run_noalloc, lutgemm_run and lutgemm_run_tc give the
    same bits."""
    q, m, n, g, batch = 3, 16384, 12288, 128, 16
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert L.tc_plan(m, n, batch, q, sms) == 1
    gen = S.generator(91)
    packed = S.draw_random_bytes(gen, L.packed_bytes(q, m, n)).to(DEV)
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02).to(DEV)
    x = S.draw_x(gen, batch, n).to(DEV)
    y_tc = L.run_tc(packed, alpha, x, m, n, q, g)
    y_run = L.run(packed, alpha, x, m, n, q, g, allow_tensor_cores=True)
    for _ in range(2):
        y = L.run_noalloc(packed, alpha, x, m, n, q, g, allow_tensor_cores=True, check=True)
        assert torch.equal(y, y_tc) and torch.equal(y, y_run)


def test_noalloc_falls_back_to_tensor_cores_when_partials_do_not_fit(L):
    """OPT-175B FC2 (12288 x 49152) at batch 8: the lookup kernel's partials
    (18.9 MB) exceed the scratch, so with the tensor cores allowed the call
    runs them with one K split (lutgemm_run_tc's bits) instead of refusing."""
    q, m, n, g, batch = 3, 12288, 49152, 128, 8
    need = batch * math.ceil(n / 1024) * math.ceil(m / 32) * 128
    assert need > (16 << 20) - 4096 - 256
    gen = S.generator(92)
    packed = S.draw_random_bytes(gen, L.packed_bytes(q, m, n)).to(DEV)
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02).to(DEV)
    x = S.draw_x(gen, batch, n).to(DEV)
    y_tc = L.run_tc(packed, alpha, x, m, n, q, g)
    for _ in range(2):
        y = L.run_noalloc(packed, alpha, x, m, n, q, g, allow_tensor_cores=True, check=True)
        assert torch.equal(y, y_tc)
    with pytest.raises(L.LutgemmError) as e:
        L.run_noalloc(packed, alpha, x, m, n, q, g)
    assert e.value.status == L.ERR_WORKSPACE


def test_noalloc_fc1_batch7_fits_and_batch8_does_not(L):
    """The scratch holds 16 MiB - 4 KiB - 256 B of partials: FC1 (49152 x
    12288) at batch 7 needs 16,515,072 B and runs; batch 8 is refused."""
    m, n, q, g = 49152, 12288, 3, 128
    cap = (16 << 20) - 4096 - 256
    need = lambda b: b * math.ceil(n / 1024) * math.ceil(m / 32) * 128
    assert need(7) <= cap < need(8)
    gen = S.generator(93)
    packed = S.draw_random_bytes(gen, L.packed_bytes(q, m, n)).to(DEV)
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02).to(DEV)
    x = S.draw_x(gen, 8, n).to(DEV)
    y_run = L.run(packed, alpha, x[:7], m, n, q, g)
    y = L.run_noalloc(packed, alpha, x[:7], m, n, q, g, check=True)
    assert torch.equal(y, y_run)
    with pytest.raises(L.LutgemmError) as e:
        L.run_noalloc(packed, alpha, x, m, n, q, g)
    assert e.value.status == L.ERR_WORKSPACE


def test_noalloc_one_slice_needs_no_scratch(L):
    """n <= 1024: the lookup kernel writes y directly, so even a problem whose
    partials would exceed the scratch runs (batch 128 x 1536 row tiles)."""
    q, m, n, g, batch = 3, 49152, 1024, 128, 128
    assert batch * math.ceil(m / 32) * 128 > (16 << 20)
    gen = S.generator(94)
    packed = S.draw_random_bytes(gen, L.packed_bytes(q, m, n)).to(DEV)
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02).to(DEV)
    x = S.draw_x(gen, batch, n).to(DEV)
    y_run = L.run(packed, alpha, x, m, n, q, g)
    y = L.run_noalloc(packed, alpha, x, m, n, q, g, check=True)
    assert torch.equal(y, y_run)


def test_noalloc_stall_is_reported_and_cleared(L):
    """A failed kernel sets the scratch's status word; lutgemm_library_status
    reports and clears it, and the next call is correct again."""
    q, m, n, g, batch = 3, 1000, 6144, 128, 2
    signs, alpha, x, _ = _inputs(707, q, m, n, g, batch, False)
    packed = L.pack_bcq(signs.to(DEV))
    a_d, x_d = alpha.to(DEV), x.to(DEV)
    L.library_status(clear=True)
    L.run_noalloc(packed, a_d, x_d, m, n, q, g, _flags=L.TEST_STALL)
    assert L.library_status(clear=True) == L.STATUS_TIMEOUT
    assert L.library_status(clear=False) == 0
    y_run = L.run(packed, a_d, x_d, m, n, q, g)
    y = L.run_noalloc(packed, a_d, x_d, m, n, q, g, check=True)
    assert torch.equal(y, y_run)


def test_noalloc_status_is_clear_after_the_parity_calls(L):
    assert L.library_status(clear=False) == 0


def test_noalloc_rejects_problems_beyond_the_scratch(L):
    """Oversized problems are refused before anything is launched.

    The pointers below are a 64-byte dummy, so every case is first checked on
    the host to need more scratch than the array holds: a call that passed
    validation would read far past them.
    """
    capacity = (16 << 20) - 4096 - 256
    small = torch.zeros(64, dtype=torch.uint8, device=DEV)
    p = ctypes.c_void_p(small.data_ptr())
    for (m, n, batch) in [(49152, 12288, 32), (12288, 49152, 8), (8192, 28672, 32)]:
        need = batch * math.ceil(n / 1024) * math.ceil(m / 32) * 32 * 4
        assert need > capacity, (m, n, batch, need)
        st = L.lib().lutgemm_run_noalloc(m, n, batch, 3, 128, p, p, None, p, p, 0, None)
        assert st == L.ERR_WORKSPACE
