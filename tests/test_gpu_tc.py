"""GPU parity of the tensor-core large-batch path (lutgemm_run_tc) against the
FP64 oracle and against the lookup path."""
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


def _problem(seed, q, m, n, g, batch):
    gen = S.generator(seed)
    signs = S.draw_signs(gen, q, m, n)
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02)
    x = S.draw_x(gen, batch, n)
    return signs, alpha, x


CASES = [
    # q, m, n, g, batch
    (3, 128, 1024, 128, 16),
    (3, 300, 2048, 128, 33),
    (2, 1000, 3072, 128, 64),
    (4, 129, 1024, 256, 130),
    (1, 512, 4096, 128, 256),
    (5, 200, 1024, 128, 300),
    (8, 64, 1024, 128, 7),
    (3, 96, 640, 128, 1),
    # last slice of 2 and of 4 pieces (units of one K block), g spanning two K blocks
    (3, 256, 1280, 128, 40),
    (2, 248, 1536, 256, 64),
    (8, 136, 2048, 128, 129),
    # g = 64: two scale groups per 128-input block (the LLaMA configs)
    (2, 256, 2048, 64, 8),
    (2, 300, 1536, 64, 40),
    (3, 128, 1024, 64, 130),
    (2, 200, 1920, 192, 33),
]


@pytest.mark.parametrize("q,m,n,g,batch", CASES)
def test_tc_matches_oracle_and_lookup_path(L, q, m, n, g, batch):
    signs, alpha, x = _problem(900 + q * 13 + batch, q, m, n, g, batch)
    packed = L.pack_bcq(signs.to(DEV))
    a_d, x_d = alpha.to(DEV), x.to(DEV)
    y_tc = L.run_tc(packed, a_d, x_d, m, n, q, g)
    y_lut = L.run(packed, a_d, x_d, m, n, q, g)
    torch.cuda.synchronize()
    y_ref = O.bcq_matmul(x.numpy(), signs.numpy(), alpha.numpy(), g)
    ok, st = compare(y_tc.cpu().numpy(), y_ref, alpha.numpy(), x.numpy(), n)
    assert ok, st
    ok2, st2 = compare(y_tc.cpu().numpy(), y_lut.cpu().numpy().astype(np.float64), alpha.numpy(), x.numpy(), n)
    assert ok2, st2


def test_tc_fp16_output_is_rounded_fp32(L):
    signs, alpha, x = _problem(950, 3, 256, 2048, 128, 40)
    packed = L.pack_bcq(signs.to(DEV))
    y32 = L.run_tc(packed, alpha.to(DEV), x.to(DEV), 256, 2048, 3, 128)
    y16 = L.run_tc(packed, alpha.to(DEV), x.to(DEV), 256, 2048, 3, 128, y_f16=True)
    torch.cuda.synchronize()
    assert torch.equal(y16, y32.to(torch.float16))


def test_tc_is_deterministic(L):
    signs, alpha, x = _problem(951, 3, 384, 3072, 128, 200)
    packed = L.pack_bcq(signs.to(DEV))
    a = L.run_tc(packed, alpha.to(DEV), x.to(DEV), 384, 3072, 3, 128)
    b = L.run_tc(packed, alpha.to(DEV), x.to(DEV), 384, 3072, 3, 128)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_tc_full_size_fc1_sampled(L):
    """OPT-175B FC1 (49152 x 12288, q = 3, g = 128) at batch 64: sampled rows."""
    m, n, q, g, batch = 49152, 12288, 3, 128, 64
    gen = S.generator(952)
    packed = S.draw_random_bytes(gen, O.packed_nbytes(q, m, n))
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02)
    x = S.draw_x(gen, batch, n)
    y = L.run_tc(packed.to(DEV), alpha.to(DEV), x.to(DEV), m, n, q, g)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(952).choice(m, 40, replace=False))
    s_rows = O.unpack_rows(packed.numpy(), q, m, n, rows)
    a_rows = alpha.numpy()[:, :, rows]
    y_ref = O.bcq_matmul_rows(x.numpy(), s_rows, a_rows, g)
    ok, st = compare(y.cpu().numpy()[:, rows], y_ref, a_rows, x.numpy(), n)
    assert ok, st


@pytest.mark.parametrize("name,m,n", [("fc2", 12288, 49152), ("qkv", 36864, 12288)])
def test_tc_full_size_bench_configuration_sampled(L, name, m, n):
    """The launch configuration bench.py --workload tc times: OPT-175B linears at
    q = 3, g = 128, batch 256 (the 128-column batch blocks): sampled rows."""
    q, g, batch = 3, 128, 256
    gen = S.generator(954 + m % 7)
    packed = S.draw_random_bytes(gen, O.packed_nbytes(q, m, n))
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02)
    x = S.draw_x(gen, batch, n)
    y = L.run_tc(packed.to(DEV), alpha.to(DEV), x.to(DEV), m, n, q, g)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(955).choice(m, 24, replace=False))
    s_rows = O.unpack_rows(packed.numpy(), q, m, n, rows)
    a_rows = alpha.numpy()[:, :, rows]
    y_ref = O.bcq_matmul_rows(x.numpy(), s_rows, a_rows, g)
    ok, st = compare(y.cpu().numpy()[:, rows], y_ref, a_rows, x.numpy(), n)
    assert ok, st


def test_tc_rejects_unsupported_shapes(L):
    signs, alpha, x = _problem(953, 3, 64, 1024, 32, 4)
    packed = L.pack_bcq(signs.to(DEV))
    with pytest.raises(L.LutgemmError) as e:            # g % 64 != 0
        L.run_tc(packed, alpha.to(DEV), x.to(DEV), 64, 1024, 3, 32)
    assert e.value.status == L.ERR_SHAPE


def test_run_with_tensor_cores_allowed_takes_the_faster_path(L):
    """lutgemm_run with LUTGEMM_ALLOW_TENSOR_CORES runs the tensor-core kernel
    (bit for bit lutgemm_run_tc's result) where its cost model expects it to
    win -- a tall matrix, many 128-row blocks per SM -- and the lookup kernel
    otherwise: a short matrix even at batch 40, any matrix below batch 8."""
    q, g = 3, 128
    # Tall: 49152 rows (384 row blocks), batch 40 and 16 (with offsets).
    m, n = 49152, 1024
    gen = S.generator(960)
    packed = S.draw_random_bytes(gen, O.packed_nbytes(q, m, n)).to(DEV)
    a_d = S.draw_alpha(gen, q, m, n, g, 0.02).to(DEV)
    x_d = S.draw_x(gen, 40, n).to(DEV)
    y = L.run(packed, a_d, x_d, m, n, q, g, allow_tensor_cores=True)
    ref = L.run_tc(packed, a_d, x_d, m, n, q, g)
    torch.cuda.synchronize()
    assert torch.equal(y, ref)
    off = (torch.randn((n // g, m), generator=S.generator(961)) * 0.01).to(DEV)
    y = L.run(packed, a_d, x_d[:16], m, n, q, g, offset=off, allow_tensor_cores=True)
    ref = L.run_tc(packed, a_d, x_d[:16], m, n, q, g, offset=off)
    torch.cuda.synchronize()
    assert torch.equal(y, ref)
    # Below batch 8: the lookup kernel.
    y = L.run(packed, a_d, x_d[:4], m, n, q, g, allow_tensor_cores=True)
    ref = L.run(packed, a_d, x_d[:4], m, n, q, g)
    torch.cuda.synchronize()
    assert torch.equal(y, ref)
    # Short: 384 rows (3 row blocks) at batch 40 -- the lookup kernel.
    m, n = 384, 2048
    signs, alpha, x = _problem(962, q, m, n, g, 40)
    packed, a_d, x_d = L.pack_bcq(signs.to(DEV)), alpha.to(DEV), x.to(DEV)
    y = L.run(packed, a_d, x_d, m, n, q, g, allow_tensor_cores=True)
    ref = L.run(packed, a_d, x_d, m, n, q, g)
    torch.cuda.synchronize()
    assert torch.equal(y, ref)
    ok, st = compare(y.cpu().numpy(), O.bcq_matmul(x.numpy(), signs.numpy(), alpha.numpy(), g),
                     alpha.numpy(), x.numpy(), n)
    assert ok, st


def test_noalloc_with_tensor_cores_allowed_needs_no_scratch(L):
    """FC1 at batch 64 needs more split-K scratch than the no-alloc array holds;
    with the tensor cores allowed it takes that path and needs none."""
    m, n, q, g, batch = 49152, 12288, 3, 128, 64
    gen = S.generator(972)
    packed = S.draw_random_bytes(gen, O.packed_nbytes(q, m, n)).to(DEV)
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02).to(DEV)
    x = S.draw_x(gen, batch, n).to(DEV)
    with pytest.raises(L.LutgemmError) as e:
        L.run_noalloc(packed, alpha, x, m, n, q, g)
    assert e.value.status == L.ERR_WORKSPACE
    y = L.run_noalloc(packed, alpha, x, m, n, q, g, allow_tensor_cores=True)
    ref = L.run_tc(packed, alpha, x, m, n, q, g)
    torch.cuda.synchronize()
    assert torch.equal(y, ref)



@pytest.mark.parametrize("q,m,n,g,batch", [(4, 256, 2048, 128, 40), (3, 300, 2560, 256, 100), (2, 128, 1024, 128, 7),
                                           (4, 136, 1280, 128, 129), (4, 256, 2048, 64, 20), (3, 96, 1536, 192, 64)])
def test_tc_uniform_weights_with_offsets(L, q, m, n, g, batch):
    """Uniform q-bit weights rewritten as BCQ plus group offsets (the lookup
    path's config of converted weights) on the tensor cores, against the
    oracle's dequantised product."""
    gen = S.generator(980 + q + batch)
    codes = torch.randint(0, 1 << q, (m, n), generator=gen, dtype=torch.uint8)
    scale = (torch.randn((n // g, m), generator=gen).abs() * 0.01).to(torch.float16)
    zero = torch.randint(0, 1 << q, (n // g, m), generator=gen, dtype=torch.uint8)
    x = S.draw_x(gen, batch, n)
    packed, alpha, offset = L.uniform_to_bcq(codes.to(DEV), scale.to(DEV), zero.to(DEV), q, g)
    y = L.run_tc(packed, alpha, x.to(DEV), m, n, q, g, offset=offset)
    torch.cuda.synchronize()
    w = O.uniform_dequant(codes.numpy(), scale.numpy(), zero.numpy(), g)
    y_ref = x.numpy().astype(np.float64) @ w.T
    ok, st = compare(y.cpu().numpy(), y_ref, alpha.cpu().numpy(), x.numpy(), n)
    assert ok, st
    # The lookup path on the same operands meets the same bound.
    y_lut = L.run(packed, alpha, x.to(DEV), m, n, q, g, offset=offset)
    torch.cuda.synchronize()
    ok, st = compare(y_lut.cpu().numpy(), y_ref, alpha.cpu().numpy(), x.numpy(), n)
    assert ok, st



@pytest.mark.parametrize("name,m,n", [("up", 28672, 8192), ("down", 8192, 28672)])
def test_tc_full_size_llama70b_sampled(L, name, m, n):
    """LLaMA-70B linears, q = 2, g = 64, batch 8 (the config's largest batch),
    x with 0.1 % outlier columns scaled x20: sampled rows against the oracle."""
    q, g, batch = 2, 64, 8
    w = S.WORKLOADS["llama70b"]
    gen = S.generator(990 + m % 11)
    packed = S.draw_random_bytes(gen, O.packed_nbytes(q, m, n))
    alpha = S.draw_alpha(gen, q, m, n, g, w.alpha_sigma)
    x = S.draw_x(gen, batch, n, outlier_frac=w.outlier_frac)
    y = L.run_tc(packed.to(DEV), alpha.to(DEV), x.to(DEV), m, n, q, g)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(991).choice(m, 24, replace=False))
    s_rows = O.unpack_rows(packed.numpy(), q, m, n, rows)
    a_rows = alpha.numpy()[:, :, rows]
    y_ref = O.bcq_matmul_rows(x.numpy(), s_rows, a_rows, g)
    ok, st = compare(y.cpu().numpy()[:, rows], y_ref, a_rows, x.numpy(), n)
    assert ok, st


@pytest.mark.parametrize("name,m,n,batch", [("fc2", 12288, 49152, 32), ("out", 12288, 12288, 16)])
def test_run_with_tensor_cores_split_k_matches_oracle(L, name, m, n, batch):
    """Short matrices: the cost model splits K over CTAs (fp32 partials in the
    workspace, the split-K reduce adds them): sampled rows against the oracle,
    and within the same bound as the single-split tensor-core result."""
    q, g = 3, 128
    gen = S.generator(995 + m % 13 + batch)
    packed = S.draw_random_bytes(gen, O.packed_nbytes(q, m, n))
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02)
    x = S.draw_x(gen, batch, n)
    p_d, a_d, x_d = packed.to(DEV), alpha.to(DEV), x.to(DEV)
    y = L.run(p_d, a_d, x_d, m, n, q, g, allow_tensor_cores=True)
    y_lut = L.run(p_d, a_d, x_d, m, n, q, g)
    torch.cuda.synchronize()
    assert not torch.equal(y, y_lut)          # not the lookup path's bits: the tensor cores ran
    rows = np.sort(np.random.default_rng(996).choice(m, 32, replace=False))
    s_rows = O.unpack_rows(packed.numpy(), q, m, n, rows)
    a_rows = alpha.numpy()[:, :, rows]
    y_ref = O.bcq_matmul_rows(x.numpy(), s_rows, a_rows, g)
    ok, st = compare(y.cpu().numpy()[:, rows], y_ref, a_rows, x.numpy(), n)
    assert ok, st
    # Deterministic: the partials are added in split order.
    y2 = L.run(p_d, a_d, x_d, m, n, q, g, allow_tensor_cores=True)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
