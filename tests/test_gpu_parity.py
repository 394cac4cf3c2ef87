"""GPU parity: the CUDA path (called through the C ABI) against the FP64 oracle.

Integer work (packing, conversion) must match bit for bit; the matmul must meet
relative L2 <= 1e-3 and |err| <= 2e-3 * sum_i mean|alpha_i| * ||x||_1 / n per
output.  Inputs come from bcq_synth (seeded); expected values come only from
the oracle.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import bcq_synth as S
from oracle import bcq_oracle as O
from tests._tol import compare, compare_f16

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def L():
    from weight_only_quantized_bcq_b200 import lutgemm
    lutgemm.lib()
    assert torch.cuda.is_available()
    return lutgemm


def _problem(seed, q, m, n, g, batch, sigma=0.02, outlier=0.0):
    gen = S.generator(seed)
    signs = S.draw_signs(gen, q, m, n)
    alpha = S.draw_alpha(gen, q, m, n, g, sigma)
    x = S.draw_x(gen, batch, n, outlier_frac=outlier)
    return signs, alpha, x


def _gpu_run(L, signs, alpha, x, g, offset=None, y_f16=False):
    q, m, n = signs.shape
    packed = L.pack_bcq(signs.to(DEV))
    y = L.run(packed, alpha.to(DEV), x.to(DEV), m, n, q, g,
              offset=None if offset is None else offset.to(DEV), y_f16=y_f16)
    torch.cuda.synchronize()
    return y.float().cpu().numpy()


# ---------------------------------------------------------------------------
# Packing and conversion: bit-exact.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("q,m,n", [(1, 32, 1024), (3, 45, 2056), (2, 70, 3000), (4, 1, 8), (3, 512, 512),
                                   (8, 33, 1032), (3, 96, 5120)])
def test_pack_bit_exact(L, q, m, n):
    signs = S.draw_signs(S.generator(100 + q), q, m, n)
    flags = torch.zeros(1, dtype=torch.int32, device=DEV)
    packed = L.pack_bcq(signs.to(DEV), status_flags=flags)
    torch.cuda.synchronize()
    want = O.pack_bcq(signs.numpy())
    got = packed.cpu().numpy()[: want.size]
    assert got.size == want.size and np.array_equal(got, want)
    assert int(flags.item()) == 0


def test_pack_flags_bad_sign(L):
    signs = S.draw_signs(S.generator(7), 2, 40, 1024)
    signs[1, 3, 17] = 0
    signs[0, 39, 1023] = 2
    flags = torch.zeros(1, dtype=torch.int32, device=DEV)
    L.pack_bcq(signs.to(DEV), status_flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) & L.FLAG_BAD_SIGN


@pytest.mark.parametrize("q,m,n,g", [(4, 96, 5120, 128), (2, 33, 1032, 8), (3, 64, 2048, 64),
                                     (1, 40, 1024, 1024), (8, 32, 1024, 256), (4, 5120, 5120, 128)])
def test_uniform_to_bcq_bit_exact(L, q, m, n, g):
    codes, scale, zero = S.draw_uniform(S.generator(200 + q), m, n, g, q, 0.01)
    flags = torch.zeros(1, dtype=torch.int32, device=DEV)
    packed, alpha, offset = L.uniform_to_bcq(codes.to(DEV), scale.to(DEV), zero.to(DEV), q, g,
                                             status_flags=flags)
    torch.cuda.synchronize()
    s_ref, a_ref, o_ref = O.uniform_to_bcq(codes.numpy(), scale.numpy(), zero.numpy(), q, g)
    want = O.pack_bcq(s_ref)
    assert np.array_equal(packed.cpu().numpy()[: want.size], want)
    assert np.array_equal(alpha.cpu().numpy().view(np.uint16), a_ref.view(np.uint16))
    assert np.array_equal(offset.cpu().numpy().view(np.uint32), o_ref.view(np.uint32))
    assert int(flags.item()) == 0


def test_uniform_flags(L):
    codes, scale, zero = S.draw_uniform(S.generator(9), 32, 1024, 128, 3, 0.01)
    codes[5, 5] = 8
    zero[2, 7] = 9
    flags = torch.zeros(1, dtype=torch.int32, device=DEV)
    L.uniform_to_bcq(codes.to(DEV), scale.to(DEV), zero.to(DEV), 3, 128, status_flags=flags)
    torch.cuda.synchronize()
    f = int(flags.item())
    assert f & L.FLAG_BAD_CODE and f & L.FLAG_BAD_ZERO


# ---------------------------------------------------------------------------
# The matmul: many (q, g, batch) combinations, several tiles, ragged tails.
# ---------------------------------------------------------------------------
CASES = [
    # q, m, n, g, batch, offset
    (3, 512, 512, 128, 1, False),      # the tiny workload
    (1, 33, 1024, 128, 1, False),
    (2, 100, 2048, 64, 2, False),
    (3, 257, 3072, 128, 3, False),
    (3, 64, 1032, 8, 1, False),         # g = 8, ragged slice
    (2, 45, 2000, 40, 1, False),        # g not a power of two
    (3, 64, 1024, 32, 1, False),
    (3, 48, 1024, 16, 2, False),
    (4, 40, 2048, 256, 2, False),       # g a multiple of 128
    (3, 70, 4096, 4096, 1, False),      # row-wise scales (g = n)
    (5, 64, 2048, 128, 1, False),       # q > 4: planes in groups of four
    (8, 33, 1024, 64, 2, False),
    (4, 96, 5120, 128, 1, True),        # offsets (converted-uniform form)
    (3, 70, 2048, 64, 2, True),
    (2, 50, 1032, 8, 1, True),
    (2, 40, 1200, 24, 1, True),
    (3, 1, 8, 8, 1, False),             # smallest shape
    (2, 31, 16, 16, 1, True),
]


@pytest.mark.parametrize("q,m,n,g,batch,with_off", CASES)
def test_run_matches_oracle(L, q, m, n, g, batch, with_off):
    signs, alpha, x = _problem(1000 + q * 7 + m, q, m, n, g, batch)
    offset = None
    if with_off:
        gen = S.generator(m + n)
        offset = (torch.randn((n // g, m), generator=gen) * 0.05).to(torch.float16).float()
    y = _gpu_run(L, signs, alpha, x, g, offset)
    y_ref = O.bcq_matmul(x.numpy(), signs.numpy(), alpha.numpy(), g,
                         None if offset is None else offset.numpy())
    ok, st = compare(y, y_ref, alpha.numpy(), x.numpy(), n)
    assert ok, st


@pytest.mark.parametrize("batch", [1, 2, 3, 4, 8, 16, 32])
def test_batch_sweep(L, batch):
    signs, alpha, x = _problem(300 + batch, 2, 128, 2048, 64, batch, sigma=0.03, outlier=0.001)
    y = _gpu_run(L, signs, alpha, x, 64)
    y_ref = O.bcq_matmul(x.numpy(), signs.numpy(), alpha.numpy(), 64)
    ok, st = compare(y, y_ref, alpha.numpy(), x.numpy(), 2048)
    assert ok, st


def test_tiny_workload(L):
    w = S.WORKLOADS["tiny"]
    sh = w.shapes[0]
    signs, alpha, x = _problem(w.seed, w.q[0], sh.m, sh.n, w.g, 1, w.alpha_sigma)
    y = _gpu_run(L, signs, alpha, x, w.g)
    y_ref = O.bcq_matmul(x.numpy(), signs.numpy(), alpha.numpy(), w.g)
    ok, st = compare(y, y_ref, alpha.numpy(), x.numpy(), sh.n)
    assert ok, st


def test_uniform4_workload(L):
    """m = n = 5120 uniform 4-bit weights rewritten as BCQ on the GPU, then multiplied."""
    w = S.WORKLOADS["uniform4"]
    sh = w.shapes[0]
    q = w.q[0]
    gen = S.generator(w.seed)
    codes, scale, zero = S.draw_uniform(gen, sh.m, sh.n, w.g, q, w.s_sigma)
    x = S.draw_x(gen, 1, sh.n)
    packed, alpha, offset = L.uniform_to_bcq(codes.to(DEV), scale.to(DEV), zero.to(DEV), q, w.g)
    y = L.run(packed, alpha, x.to(DEV), sh.m, sh.n, q, w.g, offset=offset)
    torch.cuda.synchronize()
    s_ref, a_ref, o_ref = O.uniform_to_bcq(codes.numpy(), scale.numpy(), zero.numpy(), q, w.g)
    y_ref = O.bcq_matmul(x.numpy(), s_ref, a_ref, w.g, o_ref)
    # The plain uniform product gives the same reference up to the rounding of
    # alpha_0 = s/2 for fp16-subnormal s/2 (at most 2^-25 per weight).
    y_uni = x.numpy().astype(np.float64) @ O.uniform_dequant(codes.numpy(), scale.numpy(), zero.numpy(), w.g).T
    assert np.all(np.abs(y_ref - y_uni) <= 2.0 ** -25 * np.abs(x.numpy().astype(np.float64)).sum())
    ok, st = compare(y.cpu().numpy(), y_ref, a_ref, x.numpy(), sh.n)
    assert ok, st


# ---------------------------------------------------------------------------
# Full-size shapes: random packed planes (uniform random bytes are uniform
# random +-1 bits), checked on sampled rows that the oracle computes one by one.
# ---------------------------------------------------------------------------
FULL = [
    # name, m, n, q, g, batch, sigma, outliers, seed
    ("opt175b_fc1", 49152, 12288, 3, 128, 1, 0.02, 0.0, 2),
    ("opt175b_fc2", 12288, 49152, 3, 128, 1, 0.02, 0.0, 2),
    ("llama70b_attn_b8", 8192, 8192, 2, 64, 8, 0.03, 0.001, 3),
    ("llama70b_up_b1", 28672, 8192, 2, 64, 1, 0.03, 0.001, 3),
    ("llama70b_down_b4", 8192, 28672, 2, 64, 4, 0.03, 0.001, 3),
    ("opt175b_qkv_q4_b32", 36864, 12288, 4, 128, 32, 0.02, 0.0, 4),
    ("opt175b_out_q2_b16", 12288, 12288, 2, 128, 16, 0.02, 0.0, 4),
]


def _sample_rows(m, k=48, seed=0):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(m, size=k - 4, replace=False).tolist()) | {0, 31, m - 32, m - 1}
    return np.array(sorted(rows))


@pytest.mark.parametrize("name,m,n,q,g,batch,sigma,outl,seed", FULL, ids=[f[0] for f in FULL])
def test_full_size_sampled(L, name, m, n, q, g, batch, sigma, outl, seed):
    gen = S.generator(seed)
    packed = S.draw_random_bytes(gen, O.packed_nbytes(q, m, n))
    alpha = S.draw_alpha(gen, q, m, n, g, sigma)
    x = S.draw_x(gen, batch, n, outlier_frac=outl)
    y = L.run(packed.to(DEV), alpha.to(DEV), x.to(DEV), m, n, q, g)
    torch.cuda.synchronize()
    rows = _sample_rows(m, seed=seed)
    s_rows = O.unpack_rows(packed.numpy(), q, m, n, rows)
    a_rows = alpha.numpy()[:, :, rows]
    y_ref = O.bcq_matmul_rows(x.numpy(), s_rows, a_rows, g)
    got = y.cpu().numpy()[:, rows]
    ok, st = compare(got, y_ref, a_rows, x.numpy(), n)
    assert ok, (name, st)
    assert np.all(np.isfinite(y.cpu().numpy()))


# ---------------------------------------------------------------------------
# Unit-major scales: the packing is bit-exact against the oracle, and a run
# with packed scales gives the same bits as a run with the [q][n/g][m] array.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("q,m,n,g", [(1, 32, 1024, 128), (3, 40, 2048, 128), (2, 33, 640, 128),
                                     (4, 100, 3072, 384), (5, 70, 2048, 256), (8, 33, 1152, 128),
                                     (2, 40, 2048, 64), (3, 33, 640, 64), (6, 64, 1024, 64)])
def test_pack_scales_bit_exact(L, q, m, n, g):
    alpha = S.draw_alpha(S.generator(300 + q), q, m, n, g, 0.02)
    scales = L.pack_scales(alpha.to(DEV), m, n, g)
    torch.cuda.synchronize()
    want = O.pack_scales(alpha.numpy(), g)
    assert scales.numel() == want.size
    assert np.array_equal(scales.cpu().numpy().view(np.uint16), want.view(np.uint16))


PACKED_CASES = [
    # q, m, n, g, batch, with_off, y_f16
    (3, 300, 3072, 128, 1, False, False),
    (3, 257, 2560, 256, 3, True, False),
    (1, 64, 1024, 128, 2, False, True),
    (2, 97, 640, 128, 1, True, False),
    (4, 130, 4096, 512, 4, False, False),
    (5, 70, 2048, 256, 1, False, False),
    (8, 129, 3072, 128, 2, True, True),
    (2, 300, 3072, 64, 1, False, False),      # g = 64: two scales per piece
    (2, 257, 2560, 64, 3, True, False),
    (3, 97, 640, 64, 2, False, True),
    (5, 70, 2048, 64, 1, True, False),
]


@pytest.mark.parametrize("q,m,n,g,batch,with_off,y_f16", PACKED_CASES)
def test_packed_scales_give_identical_bits(L, q, m, n, g, batch, with_off, y_f16):
    signs, alpha, x = _problem(400 + q + m, q, m, n, g, batch)
    offset = None
    if with_off:
        offset = (torch.randn((n // g, m), generator=S.generator(m + 7)) * 0.05).to(torch.float16).float().to(DEV)
    packed = L.pack_bcq(signs.to(DEV))
    a_d, x_d = alpha.to(DEV), x.to(DEV)
    scales = L.pack_scales(a_d, m, n, g)
    y_raw = L.run(packed, a_d, x_d, m, n, q, g, offset=offset, y_f16=y_f16)
    y_pk = L.run(packed, scales, x_d, m, n, q, g, offset=offset, y_f16=y_f16, scales_packed=True)
    torch.cuda.synchronize()
    assert torch.equal(y_raw, y_pk)
    y_ref = O.bcq_matmul(x.numpy(), signs.numpy(), alpha.numpy(), g,
                         None if offset is None else offset.cpu().numpy())
    if not y_f16:
        ok, st = compare(y_pk.cpu().numpy(), y_ref, alpha.numpy(), x.numpy(), n)
        assert ok, st


def test_packed_scales_full_size_fc1(L):
    """OPT-175B FC1 (49152 x 12288, q=3, g=128, batch 1) with packed scales, as
    the benchmark runs it: sampled rows against the oracle."""
    m, n, q, g, seed = 49152, 12288, 3, 128, 2
    gen = S.generator(seed)
    packed = S.draw_random_bytes(gen, O.packed_nbytes(q, m, n))
    alpha = S.draw_alpha(gen, q, m, n, g, 0.02)
    x = S.draw_x(gen, 1, n)
    scales = L.pack_scales(alpha.to(DEV), m, n, g)
    y = L.run(packed.to(DEV), scales, x.to(DEV), m, n, q, g, scales_packed=True)
    torch.cuda.synchronize()
    rows = _sample_rows(m, seed=seed)
    s_rows = O.unpack_rows(packed.numpy(), q, m, n, rows)
    a_rows = alpha.numpy()[:, :, rows]
    y_ref = O.bcq_matmul_rows(x.numpy(), s_rows, a_rows, g)
    ok, st = compare(y.cpu().numpy()[:, rows], y_ref, a_rows, x.numpy(), n)
    assert ok, st


def test_packed_scales_rejected_for_small_groups(L):
    signs, alpha, x = _problem(88, 3, 64, 1024, 32, 1)
    packed = L.pack_bcq(signs.to(DEV))
    with pytest.raises(L.LutgemmError) as e:
        L.run(packed, alpha.to(DEV), x.to(DEV), 64, 1024, 3, 32, scales_packed=True)
    assert e.value.status == L.ERR_VALUE


def test_packed_scales_full_size_llama_up_g64(L):
    """LLaMA-70B up-projection shape (28672 x 8192, q = 2, g = 64) with the
    g = 64 unit-major scales at batch 1: the same bits as the [q][n/g][m]
    scales, and sampled rows against the oracle."""
    m, n, q, g, seed = 28672, 8192, 2, 64, 3
    gen = S.generator(seed)
    packed = S.draw_random_bytes(gen, O.packed_nbytes(q, m, n)).to(DEV)
    alpha = S.draw_alpha(gen, q, m, n, g, 0.03)
    x = S.draw_x(gen, 1, n, outlier_frac=0.001)
    scales = L.pack_scales(alpha.to(DEV), m, n, g)
    y_pk = L.run(packed, scales, x.to(DEV), m, n, q, g, scales_packed=True, check=True)
    y_raw = L.run(packed, alpha.to(DEV), x.to(DEV), m, n, q, g, check=True)
    assert torch.equal(y_pk, y_raw)
    rows = _sample_rows(m, seed=seed)
    s_rows = O.unpack_rows(packed.cpu().numpy(), q, m, n, rows)
    a_rows = alpha.numpy()[:, :, rows]
    ok, st = compare(y_pk.cpu().numpy()[:, rows], O.bcq_matmul_rows(x.numpy(), s_rows, a_rows, g), a_rows,
                     x.numpy(), n)
    assert ok, st


# ---------------------------------------------------------------------------
# Output modes, determinism, workspace contract, streams.
# ---------------------------------------------------------------------------
def test_y_f16_is_rounded_fp32(L):
    signs, alpha, x = _problem(55, 3, 200, 3072, 128, 2)
    packed = L.pack_bcq(signs.to(DEV))
    ws = L.new_workspace(200, 3072, 2, 3, 128)
    y32 = L.run(packed, alpha.to(DEV), x.to(DEV), 200, 3072, 3, 128, workspace=ws)
    y16 = L.run(packed, alpha.to(DEV), x.to(DEV), 200, 3072, 3, 128, workspace=ws, y_f16=True)
    torch.cuda.synchronize()
    assert y16.dtype == torch.float16
    assert torch.equal(y16, y32.to(torch.float16))
    y_ref = O.bcq_matmul(x.numpy(), signs.numpy(), alpha.numpy(), 128)
    ok, st = compare_f16(y16.cpu().numpy(), y_ref, alpha.numpy(), x.numpy(), 3072)
    assert ok, st


def test_deterministic_and_workspace_reuse(L):
    m, n, q, g, b = 300, 6144, 3, 128, 2
    signs, alpha, x = _problem(66, q, m, n, g, b)
    packed = L.pack_bcq(signs.to(DEV))
    ws = L.new_workspace(m, n, b, q, g)
    a_d, x_d = alpha.to(DEV), x.to(DEV)
    y1 = L.run(packed, a_d, x_d, m, n, q, g, workspace=ws).clone()
    y2 = L.run(packed, a_d, x_d, m, n, q, g, workspace=ws).clone()
    x2 = S.draw_x(S.generator(67), b, n).to(DEV)
    y3 = L.run(packed, a_d, x2, m, n, q, g, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    y3_ref = O.bcq_matmul(x2.cpu().numpy(), signs.numpy(), alpha.numpy(), g)
    ok, st = compare(y3.cpu().numpy(), y3_ref, alpha.numpy(), x2.cpu().numpy(), n)
    assert ok, st
    # The status word (256 B) and the tile counters (4 KB) come first, then
    # the 256-aligned partial sums; status and counters are zero after the calls.
    ns, mt = math.ceil(n / 1024), math.ceil(m / 32)
    assert ws.numel() == 256 + 4096 + (b * ns * mt * 32 * 4 + 255) // 256 * 256
    assert not ws[: 256 + 4096].cpu().numpy().any()


def test_small_workspace_is_rejected(L):
    signs, alpha, x = _problem(77, 2, 64, 1024, 128, 1)
    packed = L.pack_bcq(signs.to(DEV))
    ws = torch.zeros(L.workspace_size(64, 1024, 1, 2, 128) - 16, dtype=torch.uint8, device=DEV)
    with pytest.raises(L.LutgemmError) as e:
        L.run(packed, alpha.to(DEV), x.to(DEV), 64, 1024, 2, 128, workspace=ws)
    assert e.value.status == L.ERR_WORKSPACE


def test_side_stream(L):
    signs, alpha, x = _problem(88, 3, 128, 2048, 128, 1)
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        packed = L.pack_bcq(signs.to(DEV))
        y = L.run(packed, alpha.to(DEV), x.to(DEV), 128, 2048, 3, 128)
    st.synchronize()
    y_ref = O.bcq_matmul(x.numpy(), signs.numpy(), alpha.numpy(), 128)
    ok, stt = compare(y.cpu().numpy(), y_ref, alpha.numpy(), x.numpy(), 2048)
    assert ok, stt
