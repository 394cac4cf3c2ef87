"""CPU checks of the Python binding's argument checks.

The library sees raw pointers only, so the binding checks each tensor's dtype,
contiguity, size and device before a call: a tensor smaller than the call's
shapes would be read or written past its end on the GPU.  These tests use CPU
tensors: a correctly sized argument gets as far as the device check ("must be
a CUDA tensor"), a wrong one is refused for its size or shape first.  Nothing
here reaches the library's compute entry points.
"""
from __future__ import annotations

import pytest
import torch


@pytest.fixture(scope="module")
def L():
    from weight_only_quantized_bcq_b200 import build, lutgemm
    build.build()
    return lutgemm


Q, M, N, G, B = 3, 64, 1024, 128, 2


def _args(L, **kw):
    a = dict(packed=torch.zeros(L.packed_bytes(Q, M, N), dtype=torch.uint8),
             alpha=torch.zeros(Q, N // G, M, dtype=torch.float16),
             x=torch.zeros(B, N, dtype=torch.float16))
    a.update(kw)
    return a


def _call(fn, a, **kw):
    return fn(a.pop("packed"), a.pop("alpha"), a.pop("x"), M, N, Q, G, **a, **kw)


@pytest.mark.parametrize("name", ["run", "run_tc", "run_noalloc"])
def test_well_formed_arguments_reach_the_device_check(L, name):
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        _call(getattr(L, name), _args(L, y=torch.zeros(B, M)))


@pytest.mark.parametrize("name", ["run", "run_tc", "run_noalloc"])
@pytest.mark.parametrize("bad,msg", [
    (dict(packed=torch.zeros(100, dtype=torch.uint8)), "packed holds 100"),
    (dict(alpha=torch.zeros(Q, N // G, M - 1, dtype=torch.float16)), "alpha holds"),
    (dict(x=torch.zeros(B, N - 8, dtype=torch.float16)), "x must be"),
    (dict(x=torch.zeros(1, B, N, dtype=torch.float16)), "x must be"),
    (dict(y=torch.zeros(B, M - 1)), "y holds"),
    (dict(y=torch.zeros(B, M, dtype=torch.float16)), "y must be a contiguous torch.float32"),
    (dict(offset=torch.zeros(N // G, M - 1)), "offset holds"),
    (dict(alpha=torch.zeros(Q, M, N // G, dtype=torch.float16).transpose(1, 2)), "alpha must be a contiguous"),
    (dict(x=torch.zeros(B, N, dtype=torch.float32)), "x must be a contiguous torch.float16"),
])
def test_product_arguments_are_checked_before_any_call(L, name, bad, msg):
    with pytest.raises(ValueError, match=msg):
        _call(getattr(L, name), _args(L, **bad))


def test_y_f16_wants_an_fp16_output(L):
    a = _args(L, y=torch.zeros(B, M))
    with pytest.raises(ValueError, match="y must be a contiguous torch.float16"):
        _call(L.run, a, y_f16=True)


def test_one_dimensional_x_is_batch_one(L):
    a = _args(L, x=torch.zeros(N, dtype=torch.float16), y=torch.zeros(1, M))
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        _call(L.run, a)
    a = _args(L, x=torch.zeros(N, dtype=torch.float16), y=torch.zeros(1, M - 1))
    with pytest.raises(ValueError, match="y holds"):
        _call(L.run, a)


def test_packed_scales_are_sized_by_the_library(L):
    need = L.scales_bytes(Q, M, N, G) // 2
    a = _args(L, alpha=torch.zeros(need - 1, dtype=torch.float16))
    with pytest.raises(ValueError, match="alpha holds"):
        _call(L.run, a, scales_packed=True)
    a = _args(L, alpha=torch.zeros(need, dtype=torch.float16), y=torch.zeros(B, M))
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        _call(L.run, a, scales_packed=True)


def test_workspace_must_be_bytes(L):
    a = _args(L, workspace=torch.zeros(L.workspace_size(M, N, B, Q, G) // 4, dtype=torch.int32))
    with pytest.raises(ValueError, match="workspace must be a contiguous torch.uint8"):
        _call(L.run, a)


def test_set_up_calls_check_their_buffers(L):
    signs = torch.ones(Q, M, N, dtype=torch.int8)
    with pytest.raises(ValueError, match="packed holds"):
        L.pack_bcq(signs, packed=torch.zeros(L.packed_bytes(Q, M, N) - 1, dtype=torch.uint8))
    with pytest.raises(ValueError, match="status_flags must be a contiguous torch.int32"):
        L.pack_bcq(signs, status_flags=torch.zeros(1, dtype=torch.int64))
    codes = torch.zeros(M, N, dtype=torch.uint8)
    scale = torch.zeros(N // G, M, dtype=torch.float16)
    zero = torch.zeros(N // G, M, dtype=torch.uint8)
    with pytest.raises(ValueError, match="scale holds"):
        L.uniform_to_bcq(codes, scale[:-1], zero, Q, G)
    with pytest.raises(ValueError, match="zero holds"):
        L.uniform_to_bcq(codes, scale, zero[:, :-1].contiguous(), Q, G)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        L.uniform_to_bcq(codes, scale, zero, Q, G)
    with pytest.raises(ValueError, match="alpha holds"):
        L.pack_scales(torch.zeros(Q, N // G, M - 1, dtype=torch.float16), M, N, G)
    with pytest.raises(ValueError, match="w must be a CUDA tensor"):
        L.fit_bcq(torch.zeros(M, N, dtype=torch.float16), Q, G)


class _FakeCuda:
    """Stands in for a CUDA tensor (only what the device check reads)."""

    def __init__(self, index):
        self.is_cuda = True
        self.device = torch.device("cuda", index)


class _FakeStream:
    def __init__(self, index):
        self.device = torch.device("cuda", index)


def test_device_check_wants_one_device_the_current_one(L, monkeypatch):
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 1)
    L._one_device(None, x=_FakeCuda(1), y=_FakeCuda(1), offset=None)
    L._one_device(_FakeStream(1), x=_FakeCuda(1))
    with pytest.raises(ValueError, match="y is on cuda:0, other arguments on cuda:1"):
        L._one_device(None, x=_FakeCuda(1), y=_FakeCuda(0))
    with pytest.raises(ValueError, match="current device is cuda:1"):
        L._one_device(None, x=_FakeCuda(0), y=_FakeCuda(0))
    with pytest.raises(ValueError, match="stream on cuda:0"):
        L._one_device(_FakeStream(0), x=_FakeCuda(1))
    with pytest.raises(ValueError, match="packed must be a CUDA tensor"):
        L._one_device(None, x=_FakeCuda(1), packed=torch.zeros(1))
