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
