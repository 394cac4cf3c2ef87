"""Host-side calls of mixed storage against the oracle (no GPU): the block
table (lutgemm_mixed_offsets), the outlier layout (lutgemm_pack_outliers), and
argument validation of the device calls, which fails before any launch."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import bcq_synth as S
from oracle import bcq_oracle as O


@pytest.fixture(scope="module")
def L():
    from weight_only_quantized_bcq_b200 import build, lutgemm
    build.build()
    lutgemm.lib()
    return lutgemm


@pytest.mark.parametrize("q_max,m,n", [(4, 40, 2048), (2, 12600, 12288), (3, 1, 8), (4, 8192, 28672)])
def test_offsets_match_oracle(L, q_max, m, n):
    lo = 1 if q_max < 4 else 2
    bp = S.draw_block_planes(S.generator(m), m, n, 0.3, lo=lo, hi=q_max)
    got = L.mixed_offsets(bp, q_max, m, n).numpy().view(np.uint32)
    assert np.array_equal(got, O.mixed_block_offsets(bp.numpy()))


def test_offsets_reject_bad_counts(L):
    bp = torch.full((2, 2), 2, dtype=torch.uint8)
    bp[1, 0] = 5
    with pytest.raises(L.LutgemmError) as e:
        L.mixed_offsets(bp, 4, 40, 2048)
    assert e.value.status == L.ERR_VALUE
    bp[1, 0] = 0
    with pytest.raises(L.LutgemmError):
        L.mixed_offsets(bp, 4, 40, 2048)
    with pytest.raises(L.LutgemmError) as e:
        L.mixed_offsets(torch.full((2, 2), 2, dtype=torch.uint8), 5, 40, 2048)
    assert e.value.status == L.ERR_SHAPE


@pytest.mark.parametrize("m,n,density", [(3, 2048, 0.3), (70, 3000, 0.02), (33, 1032, 0.1), (500, 8192, 0.005)])
def test_outlier_layout_matches_oracle(L, m, n, density):
    rp, col, val = S.draw_outliers(S.generator(n + m), m, n, density)
    optr, oent = L.pack_outliers(rp, col, val, m, n)
    w_optr, w_oent = O.pack_outliers(rp.numpy(), col.numpy(), val.numpy(), m, n)
    assert np.array_equal(optr.numpy().view(np.uint32), w_optr)
    assert np.array_equal(oent.numpy().view(np.uint32), w_oent)


def test_outlier_layout_golden(L):
    import json
    import os
    c = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "mixed_format.json")))["outlier_layout_case"]
    optr, oent = L.pack_outliers(torch.tensor(c["row_ptr"], dtype=torch.int32),
                                 torch.tensor(c["col"], dtype=torch.int32),
                                 torch.tensor(c["val"], dtype=torch.float16), c["m"], c["n"])
    assert optr.numpy().view(np.uint32).tolist() == c["optr"]
    assert oent.numpy().view(np.uint32).tolist() == c["oent"]


def test_outlier_layout_rejects_bad_csr(L):
    rp = torch.tensor([0, 2, 3], dtype=torch.int32)
    val = torch.ones(3, dtype=torch.float16)
    for col in ([5, 5, 1], [7, 2, 1], [0, 1, 4096]):          # repeated, decreasing, beyond n
        with pytest.raises(L.LutgemmError) as e:
            L.pack_outliers(rp, torch.tensor(col, dtype=torch.int32), val, 2, 2048)
        assert e.value.status == L.ERR_VALUE
    with pytest.raises(L.LutgemmError):
        L.pack_outliers(torch.tensor([0, 2, 2], dtype=torch.int32), torch.tensor([0, 1, 2], dtype=torch.int32),
                        val, 2, 2048)                          # row_ptr[m] != nnz


FAKE = 1 << 20


def _run_mixed(L, m=64, n=1024, batch=1, q_max=4, g=128, packed=FAKE, pbytes=8192, boff=FAKE, alpha=FAKE,
               optr=None, oent=None, nnz=0, x=FAKE, y=FAKE, flags=0, ws=FAKE, ws_bytes=1 << 30):
    return L.lib().lutgemm_run_mixed(m, n, batch, q_max, g, packed, pbytes, boff, alpha, optr, oent, nnz, x, y,
                                     flags, ws, ws_bytes, None)


def test_run_mixed_validation(L):
    assert _run_mixed(L, packed=None) == L.ERR_NULL
    assert _run_mixed(L, boff=None) == L.ERR_NULL
    assert _run_mixed(L, nnz=3) == L.ERR_NULL                 # outliers announced, none given
    assert _run_mixed(L, q_max=5) == L.ERR_SHAPE
    assert _run_mixed(L, q_max=0) == L.ERR_SHAPE
    assert _run_mixed(L, g=100) == L.ERR_SHAPE
    assert _run_mixed(L, flags=8) == L.ERR_VALUE                       # no such flag
    assert _run_mixed(L, g=32, flags=L.SCALES_PACKED) == L.ERR_VALUE   # unit-major scales need g % 128 == 0 or 64
    assert _run_mixed(L, alpha=FAKE + 2, flags=L.SCALES_PACKED) == L.ERR_ALIGN
    assert _run_mixed(L, pbytes=8191) == L.ERR_VALUE
    assert _run_mixed(L, boff=FAKE + 2) == L.ERR_ALIGN
    assert _run_mixed(L, x=FAKE + 8) == L.ERR_ALIGN
    assert _run_mixed(L, ws_bytes=100) == L.ERR_WORKSPACE


def test_pack_mixed_validation(L):
    lib = L.lib()
    assert lib.lutgemm_pack_bcq_mixed(None, FAKE, 4, 64, 1024, FAKE, 8192, None, None) == L.ERR_NULL
    assert lib.lutgemm_pack_bcq_mixed(FAKE, FAKE, 5, 64, 1024, FAKE, 8192, None, None) == L.ERR_SHAPE
    assert lib.lutgemm_pack_bcq_mixed(FAKE, FAKE, 4, 64, 1024, FAKE + 8, 8192, None, None) == L.ERR_ALIGN
    assert lib.lutgemm_pack_bcq_mixed(FAKE, FAKE, 4, 64, 1024, FAKE, 4096, None, None) == L.ERR_VALUE


def test_pack_scales_mixed_validation(L):
    lib = L.lib()
    assert lib.lutgemm_pack_scales_mixed(None, FAKE, 4, 64, 1024, 128, FAKE, 8192, None, None) == L.ERR_NULL
    assert lib.lutgemm_pack_scales_mixed(FAKE, FAKE, 4, 64, 1024, 32, FAKE, 8192, None, None) == L.ERR_SHAPE
    assert lib.lutgemm_pack_scales_mixed(FAKE, FAKE, 5, 64, 1024, 128, FAKE, 8192, None, None) == L.ERR_SHAPE
    assert lib.lutgemm_pack_scales_mixed(FAKE, FAKE, 4, 64, 1024, 128, FAKE + 8, 8192, None, None) == L.ERR_ALIGN
    assert lib.lutgemm_pack_scales_mixed(FAKE, FAKE, 4, 64, 1024, 128, FAKE, 8000, None, None) == L.ERR_VALUE
    assert lib.lutgemm_pack_scales_mixed(FAKE, FAKE, 4, 64, 1024, 128, FAKE, 512, None, None) == L.ERR_VALUE
