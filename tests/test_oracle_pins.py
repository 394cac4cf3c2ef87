"""Pins for the FP64 oracle: brute force, closed forms, special cases, golden fixtures.

Every check is written as a function of the oracle routine it pins, so the same
check is run once on the real routine (must pass) and once on planted mistakes
(must fail).  The planted mistakes live here, on the CPU, and only ever replace
oracle routines.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import pytest

from oracle import bcq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _fp16(rng, shape, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(np.float16)


def _alpha(rng, q, ng, m, sigma=0.02):
    return np.abs(_fp16(rng, (q, ng, m), sigma))


def _signs(rng, q, m, n):
    return (rng.integers(0, 2, size=(q, m, n)) * 2 - 1).astype(np.int8)


# ---------------------------------------------------------------------------
# Brute-force references (pure Python loops; tiny inputs only).
# ---------------------------------------------------------------------------
def _brute_y(x, signs, alpha, g, offset=None):
    q, m, n = signs.shape
    batch = x.shape[0]
    y = [[0.0] * m for _ in range(batch)]
    for b in range(batch):
        for j in range(m):
            acc = 0.0
            for k in range(n):
                w = 0.0
                for i in range(q):
                    w += float(alpha[i, k // g, j]) * int(signs[i, j, k])
                if offset is not None:
                    w += float(offset[k // g, j])
                acc += w * float(x[b, k])
            y[b][j] = acc
    return np.array(y)


def _close(a, b, rel=1e-12):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    scale = max(np.abs(b).max(initial=0.0), 1e-300)
    return a.shape == b.shape and float(np.abs(a - b).max(initial=0.0)) <= rel * scale


# ---------------------------------------------------------------------------
# Pins, each a predicate over the routine under test.
# ---------------------------------------------------------------------------
def pin_lut_table(lut_table) -> bool:
    """Table entry == explicit signed sum for all 256 patterns (exact in FP64).

    Pins bit order (bit t <-> x_t, LSB first) and sign (bit 1 <-> +1), from the
    card's 'Lookup tables instead of multiplications'.
    """
    rng = np.random.default_rng(11)
    for _ in range(4):
        x = _fp16(rng, 8).astype(np.float64)
        T = np.asarray(lut_table(x), dtype=np.float64)
        if T.shape != (256,):
            return False
        for beta in itertools.product((-1, 1), repeat=8):
            p = sum(((b + 1) // 2) << t for t, b in enumerate(beta))
            if T[p] != sum(b * v for b, v in zip(beta, x)):
                return False
    return True


def pin_matmul_bruteforce(matmul) -> bool:
    """Plain product == brute-force triple loop on tiny random problems."""
    rng = np.random.default_rng(12)
    for (q, m, n, g, batch, with_off) in [(1, 3, 16, 8, 1, False), (2, 5, 32, 16, 2, False),
                                          (3, 4, 24, 8, 2, True), (4, 6, 32, 32, 1, True),
                                          (3, 7, 40, 40, 3, False)]:
        s = _signs(rng, q, m, n)
        a = _alpha(rng, q, n // g, m)
        off = _fp16(rng, (n // g, m), 0.05).astype(np.float32) if with_off else None
        x = _fp16(rng, (batch, n))
        if not _close(matmul(x, s, a, g, off), _brute_y(x, s, a, g, off)):
            return False
    return True


def pin_q1_textbook(matmul) -> bool:
    """q=1, alpha=1, no offset: the textbook +-1 matvec, exact on integer x."""
    rng = np.random.default_rng(13)
    m, n = 9, 64
    s = _signs(rng, 1, m, n)
    a = np.ones((1, 1, m), dtype=np.float16)
    xi = rng.integers(-5, 6, size=(2, n))
    x = xi.astype(np.float16)
    want = [[sum(int(s[0, j, k]) * int(xi[b, k]) for k in range(n)) for j in range(m)] for b in range(2)]
    return np.array_equal(np.asarray(matmul(x, s, a, n, None)), np.array(want, dtype=np.float64))


def pin_one_hot(matmul) -> bool:
    """One-hot x returns the dequantised column exactly."""
    rng = np.random.default_rng(14)
    q, m, n, g = 3, 6, 32, 8
    s = _signs(rng, q, m, n)
    a = _alpha(rng, q, n // g, m)
    off = _fp16(rng, (n // g, m), 0.05).astype(np.float32)
    for k in (0, 7, 8, 31):
        x = np.zeros((1, n), dtype=np.float16)
        x[0, k] = 1.0
        y = np.asarray(matmul(x, s, a, g, off))[0]
        col = [sum(float(a[i, k // g, j]) * int(s[i, j, k]) for i in range(q)) + float(off[k // g, j])
               for j in range(m)]
        if not np.array_equal(y, np.array(col)):
            return False
    return True


def pin_all_plus(matmul) -> bool:
    """All signs +1: y = sum_G sum_i alpha[i,G,j] * S_G with S_G the group's x-sum."""
    rng = np.random.default_rng(15)
    q, m, n, g = 2, 5, 64, 16
    s = np.ones((q, m, n), dtype=np.int8)
    a = _alpha(rng, q, n // g, m)
    x = _fp16(rng, (2, n))
    SG = x.astype(np.float64).reshape(2, n // g, g).sum(axis=2)        # [b][G]
    want = np.einsum("bG,iGj->bj", SG, a.astype(np.float64))
    return _close(matmul(x, s, a, g, None), want)


def pin_row_wise(matmul) -> bool:
    """g = n (row-wise scales): y = sum_i alpha_i * (B_i x)."""
    rng = np.random.default_rng(16)
    q, m, n = 3, 7, 48
    s = _signs(rng, q, m, n)
    a = _alpha(rng, q, 1, m)
    x = _fp16(rng, (1, n))
    want = sum(a[i, 0].astype(np.float64) * (s[i].astype(np.float64) @ x[0].astype(np.float64))
               for i in range(q))
    return _close(np.asarray(matmul(x, s, a, n, None))[0], want)


def pin_uniform_golden(uniform_to_bcq) -> bool:
    """Hand-worked uniform->BCQ examples (tests/golden/uniform_to_bcq_examples.json)."""
    for case in _golden("uniform_to_bcq_examples.json")["cases"]:
        q, g = case["q"], case["g"]
        codes = np.array([case["codes"]], dtype=np.uint8)
        scale = np.array([[case["s"]]], dtype=np.float16)
        zero = np.array([[case["z"]]], dtype=np.uint8)
        signs, alpha, offset = uniform_to_bcq(codes, scale, zero, q, g)
        if not np.array_equal(np.asarray(signs)[:, 0, :], np.array(case["signs"], dtype=np.int8)):
            return False
        if not np.array_equal(np.asarray(alpha, dtype=np.float64)[:, 0, 0], np.array(case["alpha"])):
            return False
        if float(np.asarray(offset)[0, 0]) != case["offset"]:
            return False
        w = O.dequantize_bcq(signs, alpha, g, offset)[0]
        if not np.array_equal(w, np.array(case["w"])):
            return False
    return True


def pin_uniform_closed_form(uniform_to_bcq) -> bool:
    """Every (q, c, z): the BCQ rewrite dequantises to s*(c - z) exactly (s >= 2^-13)."""
    rng = np.random.default_rng(17)
    for q in (1, 2, 3, 4):
        top = 1 << q
        cs, zs = np.meshgrid(np.arange(top), np.arange(top), indexing="ij")
        cs, zs = cs.reshape(-1), zs.reshape(-1)
        m = cs.size
        g = 8
        codes = np.repeat(cs[:, None], g, axis=1).astype(np.uint8)               # [m][8]
        scale = np.abs(_fp16(rng, (1, m), 0.01)).astype(np.float16)
        scale = np.maximum(scale, np.float16(2.0 ** -13))
        zero = zs[None, :].astype(np.uint8)
        signs, alpha, offset = uniform_to_bcq(codes, scale, zero, q, g)
        w = O.dequantize_bcq(signs, alpha, g, offset)
        want = scale.astype(np.float64)[0][:, None] * (cs[:, None] - zs[:, None]).astype(np.float64)
        if not np.array_equal(w, np.repeat(want, g, axis=1)):
            return False
    return True


def _golden_packed(case):
    buf = np.zeros(case["total_bytes"], dtype=np.uint8)
    for off, val in case["nonzero"].items():
        buf[int(off)] = val
    return buf


def pin_pack_golden(pack_bcq) -> bool:
    """Single-bit and padding fixtures derived by hand from the layout text."""
    gold = _golden("pack_layout_single_bits.json")
    for case in gold["cases"]:
        q, m, n = case["q"], case["m"], case["n"]
        s = -np.ones((q, m, n), dtype=np.int8)
        i, r, k = case["plus_one"]
        s[i, r, k] = 1
        # All -1 rows give zero bytes; only the single +1 sets a bit.
        if not np.array_equal(np.asarray(pack_bcq(s)), _golden_packed(case)):
            return False
    pc = gold["all_plus_padding_case"]
    s = np.ones((pc["q"], pc["m"], pc["n"]), dtype=np.int8)
    want = np.zeros(pc["total_bytes"], dtype=np.uint8)
    want[pc["nonzero_offsets"]] = pc["value"]
    return np.array_equal(np.asarray(pack_bcq(s)), want)


def pin_unpack_golden(unpack_bcq) -> bool:
    gold = _golden("pack_layout_single_bits.json")
    for case in gold["cases"]:
        q, m, n = case["q"], case["m"], case["n"]
        s = np.asarray(unpack_bcq(_golden_packed(case), q, m, n))
        want = -np.ones((q, m, n), dtype=np.int8)
        i, r, k = case["plus_one"]
        want[i, r, k] = 1
        if not np.array_equal(s, want):
            return False
    return True


# ---------------------------------------------------------------------------
# The pins on the real oracle.
# ---------------------------------------------------------------------------
def test_lut_table_pinned():
    assert pin_lut_table(O.lut_table)


def test_lut_table_invariants():
    rng = np.random.default_rng(3)
    x = _fp16(rng, 8).astype(np.float64)
    T = O.lut_table(x)
    assert T[0] == -x.sum() and T[255] == x.sum()
    assert np.array_equal(T, -T[::-1])                      # T[p] = -T[255 - p]
    for t in range(8):
        assert T[1 << t] - T[0] == 2 * x[t]


@pytest.mark.parametrize("fn", ["bcq_matmul", "lut_matmul"])
def test_matmul_pins(fn):
    f = getattr(O, fn)
    assert pin_matmul_bruteforce(f)
    assert pin_q1_textbook(f)
    assert pin_one_hot(f)
    assert pin_all_plus(f)
    assert pin_row_wise(f)


def test_lut_matmul_equals_plain_product_random():
    """The lookup regrouping reaches the plain product (card: 'no dequantization is needed')."""
    rng = np.random.default_rng(21)
    for (q, m, n, g, batch) in [(3, 33, 256, 128, 2), (2, 17, 192, 64, 3), (4, 8, 64, 8, 1)]:
        s = _signs(rng, q, m, n)
        a = _alpha(rng, q, n // g, m)
        off = _fp16(rng, (n // g, m), 0.05).astype(np.float32)
        x = _fp16(rng, (batch, n))
        assert _close(O.lut_matmul(x, s, a, g, off), O.bcq_matmul(x, s, a, g, off), 1e-12)


def test_uniform_pins():
    assert pin_uniform_golden(O.uniform_to_bcq)
    assert pin_uniform_closed_form(O.uniform_to_bcq)


def test_uniform_dequant_golden():
    for case in _golden("uniform_to_bcq_examples.json")["cases"]:
        w = O.uniform_dequant(np.array([case["codes"]], dtype=np.uint8),
                              np.array([[case["s"]]], dtype=np.float16),
                              np.array([[case["z"]]], dtype=np.uint8), case["g"])
        assert np.array_equal(w[0], np.array(case["w"]))


def test_uniform_subnormal_scale_within_half_ulp():
    """s*2^-1 below the fp16 normal range may round; error <= 2^-25 per weight."""
    q, g = 4, 8
    s = np.array([[2.0 ** -14 + 2.0 ** -24, 2.0 ** -20 + 2.0 ** -24]], dtype=np.float16)
    codes = np.tile(np.arange(8, dtype=np.uint8), (2, 1))
    zero = np.array([[3, 11]], dtype=np.uint8)
    signs, alpha, offset = O.uniform_to_bcq(codes, s, zero, q, g)
    w = O.dequantize_bcq(signs, alpha, g, offset)
    want = O.uniform_dequant(codes, s, zero, g)
    assert float(np.abs(w - want).max()) <= 2.0 ** -25


def test_uniform_rejects_out_of_range():
    with pytest.raises(ValueError):
        O.uniform_to_bcq(np.full((1, 8), 4, np.uint8), np.ones((1, 1), np.float16),
                         np.zeros((1, 1), np.uint8), 2, 8)
    with pytest.raises(ValueError):
        O.uniform_to_bcq(np.zeros((1, 8), np.uint8), np.ones((1, 1), np.float16),
                         np.full((1, 1), 4, np.uint8), 2, 8)


def test_uniform_matmul_matches_plain_uniform():
    rng = np.random.default_rng(22)
    q, m, n, g = 4, 12, 256, 64
    codes = rng.integers(0, 16, size=(m, n)).astype(np.uint8)
    scale = np.maximum(np.abs(_fp16(rng, (n // g, m), 0.01)), np.float16(2.0 ** -13)).astype(np.float16)
    zero = rng.integers(0, 16, size=(n // g, m)).astype(np.uint8)
    x = _fp16(rng, (2, n))
    signs, alpha, offset = O.uniform_to_bcq(codes, scale, zero, q, g)
    want = x.astype(np.float64) @ O.uniform_dequant(codes, scale, zero, g).T
    assert _close(O.bcq_matmul(x, signs, alpha, g, offset), want, 1e-12)
    assert _close(O.lut_matmul(x, signs, alpha, g, offset), want, 1e-12)


def test_pack_pins():
    assert pin_pack_golden(O.pack_bcq)
    assert pin_unpack_golden(O.unpack_bcq)


@pytest.mark.parametrize("q,m,n", [(1, 32, 1024), (3, 45, 2056), (2, 70, 3000), (4, 1, 8)])
def test_pack_roundtrip(q, m, n):
    rng = np.random.default_rng(q * 1000 + m)
    s = _signs(rng, q, m, n)
    pk = O.pack_bcq(s)
    assert pk.size == O.packed_nbytes(q, m, n)
    assert np.array_equal(O.unpack_bcq(pk, q, m, n), s)
    rows = np.array([0, m - 1, m // 2])
    assert np.array_equal(O.unpack_rows(pk, q, m, n, rows), s[:, rows, :])


def test_vectorised_unpack_pins():
    assert pin_unpack_golden(O.unpack_bcq_vec)


@pytest.mark.parametrize("q,m,n", [(1, 32, 1024), (3, 45, 2056), (2, 70, 3000), (4, 1, 8), (8, 33, 1032)])
def test_vectorised_unpack_equals_loop_unpack(q, m, n):
    rng = np.random.default_rng(q * 77 + m)
    s = _signs(rng, q, m, n)
    pk = O.pack_bcq(s)
    assert np.array_equal(O.unpack_bcq_vec(pk, q, m, n), s)
    assert np.array_equal(O.unpack_bcq_vec(pk, q, m, n), O.unpack_bcq(pk, q, m, n))


@pytest.mark.parametrize("q,m,n,R0,R1", [(3, 100, 2056, 1, 3), (2, 100, 2056, 2, 4), (1, 64, 1024, 0, 2),
                                          (4, 33, 8, 1, 2)])
def test_packed_row_tiles_is_the_packed_sub_matrix(q, m, n, R0, R1):
    rng = np.random.default_rng(q + m + R0)
    s = _signs(rng, q, m, n)
    sub, m_sub = O.packed_row_tiles(O.pack_bcq(s), q, m, n, R0, R1)
    rows = s[:, 32 * R0: 32 * R0 + m_sub]
    assert m_sub == rows.shape[1]
    assert np.array_equal(sub, O.pack_bcq(rows))
    assert np.array_equal(O.unpack_bcq_vec(sub, q, m_sub, n), rows)


def _unpack_vec_msb_first(packed, q, m, n):
    # Bit order reversed inside each byte: must fail the golden single bits.
    pk = np.asarray(packed, dtype=np.uint8)
    rev = np.unpackbits(pk[:, None], axis=1, bitorder="little")
    return O.unpack_bcq_vec(np.packbits(rev, axis=1, bitorder="big").reshape(-1), q, m, n)


def _unpack_vec_no_half_swap(packed, q, m, n):
    # Lanes 16..31 read the same piece as lanes 0..15.
    pk = np.asarray(packed, dtype=np.uint8).reshape(-1)
    ns, mt = math.ceil(n / 1024), math.ceil(m / 32)
    ch = pk.reshape(ns, mt, 8, q, 32, 16).copy()
    ch[:, :, :, :, 16:, :] = ch[:, :, [4, 5, 6, 7, 0, 1, 2, 3], :, 16:, :]
    return O.unpack_bcq_vec(ch.reshape(-1), q, m, n)


@pytest.mark.parametrize("mutant", [_unpack_vec_msb_first, _unpack_vec_no_half_swap])
def test_vectorised_unpack_pins_catch_mistakes(mutant):
    assert not pin_unpack_golden(mutant)


def test_pack_rejects_non_sign_values():
    s = np.ones((1, 4, 8), dtype=np.int8)
    s[0, 1, 3] = 0
    with pytest.raises(ValueError):
        O.pack_bcq(s)


# ---------------------------------------------------------------------------
# Planted mistakes: each must make at least one pin fail.
# ---------------------------------------------------------------------------
def _lut_msb_first(x):
    x = np.asarray(x, dtype=np.float64)
    return O.lut_table(x[::-1])


def _lut_sign_flipped(x):
    return -O.lut_table(x)


def _lut_dropped_term(x):
    x = np.array(x, dtype=np.float64)
    x[7] = 0.0
    return O.lut_table(x)


@pytest.mark.parametrize("mutant", [_lut_msb_first, _lut_sign_flipped, _lut_dropped_term])
def test_lut_pin_catches_mistakes(mutant):
    assert not pin_lut_table(mutant)


def _mm_no_offset(x, s, a, g, off=None):
    return O.bcq_matmul(x, s, a, g, None)


def _mm_group_shift(x, s, a, g, off=None):
    return O.bcq_matmul(x, s, np.roll(np.asarray(a), 1, axis=1), g, off)


def _mm_alpha_layout_confused(x, s, a, g, off=None):
    # alpha read as [q][m][n/g] instead of [q][n/g][m]
    a = np.asarray(a)
    q, ng, m = a.shape
    return O.bcq_matmul(x, s, a.reshape(q, m, ng).transpose(0, 2, 1), g, off)


def _mm_plane_dropped(x, s, a, g, off=None):
    a2 = np.array(a, dtype=np.float64)
    if a2.shape[0] > 1:
        a2[-1] = 0.0
    else:
        a2 = a2 * 0.5
    return O.bcq_matmul(x, s, a2, g, off)


def _mm_sign_flipped(x, s, a, g, off=None):
    return O.bcq_matmul(x, -np.asarray(s), a, g, off)


@pytest.mark.parametrize("mutant", [_mm_no_offset, _mm_group_shift, _mm_alpha_layout_confused,
                                    _mm_plane_dropped, _mm_sign_flipped])
def test_matmul_pins_catch_mistakes(mutant):
    pins = (pin_matmul_bruteforce, pin_q1_textbook, pin_one_hot, pin_all_plus, pin_row_wise)
    assert not all(p(mutant) for p in pins)


def _uni_no_half(codes, scale, zero, q, g):
    s, a, o = O.uniform_to_bcq(codes, scale, zero, q, g)
    return s, (np.asarray(a, dtype=np.float64) * 2).astype(np.float16), o


def _uni_offset_sign(codes, scale, zero, q, g):
    s, a, o = O.uniform_to_bcq(codes, scale, zero, q, g)
    return s, a, -o


def _uni_plane_order(codes, scale, zero, q, g):
    s, a, o = O.uniform_to_bcq(codes, scale, zero, q, g)
    return s[::-1].copy(), a, o


@pytest.mark.parametrize("mutant", [_uni_no_half, _uni_offset_sign, _uni_plane_order])
def test_uniform_pins_catch_mistakes(mutant):
    assert not (pin_uniform_golden(mutant) and pin_uniform_closed_form(mutant))


def test_pack_pins_catch_wrong_piece_rotation(monkeypatch):
    monkeypatch.setattr(O, "_piece_and_run", lambda U, l, j: (U, j ^ (l % 16)))
    assert not pin_pack_golden(O.pack_bcq)


def test_pack_pins_catch_wrong_run_xor(monkeypatch):
    monkeypatch.setattr(O, "_piece_and_run", lambda U, l, j: (U ^ (4 * (l // 16)), j))
    assert not pin_pack_golden(O.pack_bcq)


def test_pack_pins_catch_plane_major_chunk_order():
    def plane_major(s):
        q, m, n = s.shape
        pk = O.pack_bcq(s)
        ns, mt = -(-n // 1024), -(-m // 32)
        return pk.reshape(ns, mt, 8, q, 512).transpose(0, 1, 3, 2, 4).reshape(-1)
    assert not pin_pack_golden(plane_major)


def test_pack_pins_catch_msb_first():
    def msb_first(s):
        bits = np.unpackbits(O.pack_bcq(s), bitorder="little")
        return np.packbits(bits, bitorder="big")
    assert not pin_pack_golden(msb_first)


# ---------------------------------------------------------------------------
# The footprint the card prints (Key points: 347.9 GB -> 65.3 GB, 5.33x) pins
# the bits-per-weight count used for algorithmic bytes.
# ---------------------------------------------------------------------------
# ---------------------------------------------------------------------------
# Unit-major scale layout: hand-derived positions (tests/golden), round trip,
# and planted mistakes in the index map.
# ---------------------------------------------------------------------------
def _distinct_alpha(q, ng, m):
    """fp16 scales whose bit patterns are 1, 2, 3, ... (all distinct, none zero)."""
    bits = np.arange(1, q * ng * m + 1, dtype=np.uint16).reshape(q, ng, m)
    return bits.view(np.float16)


def pin_scales_golden(pack_scales) -> bool:
    for case in _golden("scales_layout_positions.json")["cases"]:
        q, m, n, g = case["q"], case["m"], case["n"], case["g"]
        alpha = _distinct_alpha(q, n // g, m)
        out = np.asarray(pack_scales(alpha, g), dtype=np.float16).view(np.uint16)
        if out.size != case["nelem"] or out.size * 2 != O.scales_nbytes(q, m, n, g):
            return False
        for e in case["entries"]:
            want = 0 if e[1] is None else int(alpha.view(np.uint16)[e[1], e[2], e[3]])
            if int(out[e[0]]) != want:
                return False
    return True


def test_scales_pins():
    assert pin_scales_golden(O.pack_scales)


@pytest.mark.parametrize("q,m,n,g", [(1, 32, 1024, 128), (3, 40, 2048, 128), (4, 100, 3072, 384),
                                     (5, 70, 2048, 256), (8, 33, 1152, 128), (2, 33, 640, 128),
                                     (2, 40, 2048, 64), (3, 33, 640, 64), (6, 64, 1024, 64)])
def test_scales_roundtrip(q, m, n, g):
    alpha = _distinct_alpha(q, n // g, m)
    packed = O.pack_scales(alpha, g)
    assert packed.size * 2 == O.scales_nbytes(q, m, n, g)
    back = O.unpack_scales(packed, q, m, n, g)
    assert np.array_equal(back.view(np.uint16), alpha.view(np.uint16))
    # Every stored value is a scale or padding zero, and each scale is stored
    # once per piece of its group that lies inside n.
    vals = packed.view(np.uint16)
    counts = np.bincount(vals, minlength=alpha.size + 1)
    assert np.all(counts[1:] == max(1, g // 128))


def test_scales_reject_groups_below_half_a_piece():
    with pytest.raises(ValueError):
        O.scales_nbytes(3, 32, 1024, 32)
    with pytest.raises(ValueError):
        O.scales_nbytes(3, 32, 1024, 192)


def _scales_pieces_not_swapped(alpha, g):
    """Planted: lanes 16..31 read the same piece as lanes 0..15."""
    a = np.asarray(alpha, dtype=np.float16)
    q, ng, m = a.shape
    n = ng * g
    ns, mt, sp, npg = math.ceil(n / 1024), math.ceil(m / 32), min(q, 4), math.ceil(q / 4)
    out = np.zeros((ns, mt, npg, 32, 8, sp), dtype=np.float16)
    for s_ in range(ns):
        for U in range(8):
            k0 = 1024 * s_ + 128 * U
            if k0 >= n:
                continue
            for i in range(q):
                col = np.zeros(mt * 32, dtype=np.float16)
                col[:m] = a[i, k0 // g, :]
                out[s_, :, i // 4, :, U, i % 4] = col.reshape(mt, 32)
    return out.reshape(-1)


def _scales_step_major(alpha, g):
    """Planted: step outside lane ([..][U][l][e] instead of [..][l][U][e])."""
    good = O.pack_scales(alpha, g)
    a = np.asarray(alpha)
    q, ng, m = a.shape
    n = ng * g
    ns, mt, sp, npg = math.ceil(n / 1024), math.ceil(m / 32), min(q, 4), math.ceil(q / 4)
    return good.reshape(ns, mt, npg, 32, 8, sp).transpose(0, 1, 2, 4, 3, 5).reshape(-1)


def _scales_planes_reversed(alpha, g):
    """Planted: planes stored in reverse order."""
    return O.pack_scales(np.asarray(alpha)[::-1], g)


def _scales_group_per_run(alpha, g):
    """Planted: group index taken from the run (8 inputs) instead of the piece."""
    a = np.asarray(alpha, dtype=np.float16)
    q, ng, m = a.shape
    n = ng * g
    ns, mt, sp, npg = math.ceil(n / 1024), math.ceil(m / 32), min(q, 4), math.ceil(q / 4)
    out = np.zeros((ns, mt, npg, 32, 8, sp), dtype=np.float16)
    for s_ in range(ns):
        for U in range(8):
            for half in range(2):
                P = U ^ (4 * half)
                k0 = 1024 * s_ + 8 * P
                if 1024 * s_ + 128 * P >= n:
                    continue
                for i in range(q):
                    col = np.zeros(mt * 32, dtype=np.float16)
                    col[:m] = a[i, k0 // g, :]
                    ln = slice(16 * half, 16 * half + 16)
                    out[s_, :, i // 4, ln, U, i % 4] = col.reshape(mt, 32)[:, ln]
    return out.reshape(-1)


def _scales_halves_swapped(alpha, g):
    # g = 64: the two halves of a piece in the wrong order.
    out = O.pack_scales(alpha, g)
    if g == 64:
        out = out.reshape(-1, 2)[:, ::-1].reshape(-1).copy()
    return out


@pytest.mark.parametrize("mutant", [_scales_halves_swapped, _scales_pieces_not_swapped, _scales_step_major, _scales_planes_reversed,
                                    _scales_group_per_run])
def test_scales_pins_catch_mistakes(mutant):
    assert not pin_scales_golden(mutant)


def test_footprint_matches_printed_ratio():
    from weight_only_quantized_bcq_b200.roofline import bits_per_weight
    gold = _golden("opt175b_footprint.json")
    ratio = 16.0 / bits_per_weight(gold["q"], gold["g_row"])
    assert round(ratio, 2) == gold["ratio"]
    assert abs(gold["fp16_gb"] / gold["lutgemm_gb"] - ratio) < 0.01
    # g = 128 would not reproduce it (4.74x): the count is sensitive to the scale term.
    assert round(16.0 / bits_per_weight(3, 128), 2) == 4.74


# ---------------------------------------------------------------------------
# BCQ fitting (greedy + alternating least squares): closed forms, exact
# recovery of representable weights, brute force on tiny cases, monotone
# error, and planted mistakes.
# ---------------------------------------------------------------------------
def _fp16_weights(rng, m, n, sigma=0.02):
    return (rng.standard_normal((m, n)) * sigma).astype(np.float16)


def pin_fit_q1_closed_form(fit_bcq) -> bool:
    """q = 1: beta = sign(w) (0 -> +1), alpha = fp16(mean |w|), for any iters."""
    rng = np.random.default_rng(11)
    w = _fp16_weights(rng, 6, 256)
    w[0, :5] = 0
    for iters in (0, 2):
        signs, alpha, _ = fit_bcq(w, 1, 64, iters)
        want_s = np.where(w.astype(np.float64) >= 0, 1, -1)
        want_a = np.abs(w.astype(np.float64)).reshape(6, 4, 64).mean(-1).astype(np.float16).T
        if not (np.array_equal(signs[0], want_s) and np.array_equal(alpha[0].view(np.uint16),
                                                                    want_a.view(np.uint16))):
            return False
    return True


def _representable(rng, m, ng, g):
    """w = c * (b1 + b2/2 + b3/4) per group, c a power of two: exact in fp16."""
    c = 2.0 ** rng.integers(-9, -4, size=(m, ng))
    b = rng.choice([-1.0, 1.0], size=(3, m, ng, g))
    w = c[..., None] * (b[0] + b[1] / 2 + b[2] / 4)
    return w.reshape(m, ng * g).astype(np.float16), b, c


def pin_fit_exact_recovery(fit_bcq) -> bool:
    rng = np.random.default_rng(12)
    w, b, c = _representable(rng, 5, 3, 128)
    signs, alpha, err = fit_bcq(w, 3, 128, 3)
    want_a = np.stack([c, c / 2, c / 4]).transpose(0, 2, 1)
    return (np.array_equal(signs.reshape(3, 5, 3, 128), b.astype(np.int8))
            and np.array_equal(alpha.astype(np.float64), want_a) and float(np.abs(err).max()) == 0.0)


def pin_fit_q1_global_optimum(fit_bcq) -> bool:
    """q = 1, g = 8: the fit's error equals the brute-force minimum over all 256 sign vectors."""
    rng = np.random.default_rng(13)
    w = _fp16_weights(rng, 3, 8, 1.0)
    _, alpha, err = fit_bcq(w, 1, 8, 2)
    for j in range(3):
        wj = w[j].astype(np.float64)
        best = min(float(((wj - (s @ wj) / 8 * np.array(s)) ** 2).sum())
                   for s in itertools.product([-1.0, 1.0], repeat=8))
        # the fit stores alpha in fp16, so its error may exceed the exact optimum by the rounding
        a = float(alpha[0, 0, j])
        if not (best - 1e-12 <= err[0, j] <= best + 8 * abs(a - np.abs(wj).mean()) * np.abs(wj).sum() + 1e-12):
            return False
    return True


def pin_nearest_codes_bruteforce(nearest_codes) -> bool:
    rng = np.random.default_rng(14)
    q, g = 3, 16
    w = rng.standard_normal((4, g))
    a = np.abs(rng.standard_normal((q, 4))) + 0.1
    got = nearest_codes(w, a)
    for r in range(4):
        for k in range(g):
            best, arg = None, None
            for s in itertools.product([-1.0, 1.0], repeat=q):
                v = sum(a[i, r] * s[i] for i in range(q))
                if best is None or abs(w[r, k] - v) < best:
                    best, arg = abs(w[r, k] - v), s
            if tuple(got[:, r, k]) != arg:
                return False
    return True


def pin_fit_stored_signs_are_best(fit_bcq) -> bool:
    """Every stored sign combination is a nearest one for the stored fp16 scales
    (brute force over the 2^q combinations), and the returned error is the
    error of the stored result."""
    rng = np.random.default_rng(18)
    q, g, m, n = 3, 128, 24, 512
    w = _fp16_weights(rng, m, n)
    signs, alpha, err = fit_bcq(w, q, g, 2)
    combos = np.array(list(itertools.product([-1.0, 1.0], repeat=q)))      # [8][q]
    for j in range(m):
        for G in range(n // g):
            a = alpha[:, G, j].astype(np.float64)
            vals = combos @ a
            wk = w[j, G * g:(G + 1) * g].astype(np.float64)
            v = np.einsum("i,ik->k", a, signs[:, j, G * g:(G + 1) * g].astype(np.float64))
            best = np.abs(wk[:, None] - vals[None, :]).min(axis=1)
            if np.any(np.abs(wk - v) > best + 1e-15):
                return False
            e = float(((wk - v) ** 2).sum())
            if abs(e - err[G, j]) > 1e-12 * max(e, 1e-30):
                return False
    return True


def test_fit_pins():
    assert pin_fit_stored_signs_are_best(O.fit_bcq)
    assert pin_fit_q1_closed_form(O.fit_bcq)
    assert pin_fit_exact_recovery(O.fit_bcq)
    assert pin_fit_q1_global_optimum(O.fit_bcq)
    assert pin_nearest_codes_bruteforce(O.nearest_codes)


@pytest.mark.parametrize("q,g", [(2, 64), (3, 128), (4, 128), (3, 8)])
def test_fit_error_never_rises(q, g):
    rng = np.random.default_rng(15 + q)
    w = _fp16_weights(rng, 7, 512)
    trace = O.fit_bcq_trace(w, q, g, 4)
    scale = (w.astype(np.float64).reshape(7, -1, g) ** 2).sum(-1)
    for before, after in zip(trace, trace[1:]):
        assert np.all(after <= before + 1e-12 * scale)
    assert np.all(trace[-1] < trace[0] + 1e-12 * scale)


def test_alpha_step_matches_least_squares():
    """The Cholesky alpha-step against numpy's least-squares solver."""
    rng = np.random.default_rng(16)
    q, g = 4, 64
    B = rng.choice([-1.0, 1.0], size=(q, 9, g))
    w = rng.standard_normal((9, g))
    a = O._ls_alpha(w, B, np.zeros((q, 9)), g)
    for r in range(9):
        ref = np.linalg.lstsq(B[:, r, :].T, w[r], rcond=None)[0]
        assert np.allclose(a[:, r], ref, rtol=1e-10, atol=1e-12)


def test_alpha_step_keeps_alpha_for_dependent_planes():
    rng = np.random.default_rng(17)
    B = rng.choice([-1.0, 1.0], size=(2, 1, 32))
    B[1] = -B[0]                                   # plane 1 = -plane 0: singular normal matrix
    old = np.array([[0.3], [0.2]])
    a = O._ls_alpha(rng.standard_normal((1, 32)), B, old, 32)
    assert np.array_equal(a, old)


def _fit_no_residual(w, q, g, iters):
    """Planted: the greedy pass never subtracts the fitted plane."""
    W = np.asarray(w, dtype=np.float64)
    m, n = W.shape
    Wg = W.reshape(m, n // g, g)
    B = np.stack([np.where(Wg >= 0, 1.0, -1.0)] * q)
    a = np.stack([np.abs(Wg).mean(-1)] * q)
    for _ in range(iters):
        a = O._ls_alpha(Wg, B, a, g)
        B = O.nearest_codes(Wg, a)
    a16 = a.astype(np.float16)
    B = O.nearest_codes(Wg, a16.astype(np.float64))
    err = ((Wg - np.einsum("i...,i...k->...k", a16.astype(np.float64), B)) ** 2).sum(-1)
    return B.reshape(q, m, n).astype(np.int8), np.transpose(a16, (0, 2, 1)), err.T


def _fit_alpha_not_rounded_for_signs(w, q, g, iters):
    """Planted: alpha rounded to fp16 after the signs were chosen with the exact alpha."""
    Wg, a, B = O._fit_groups(w, q, g, iters)
    a16 = a.astype(np.float16)
    err = ((Wg - np.einsum("i...,i...k->...k", a16.astype(np.float64), B)) ** 2).sum(-1)
    m, ng, _ = Wg.shape
    return B.reshape(q, m, ng * g).astype(np.int8), np.transpose(a16, (0, 2, 1)), err.T


def _nearest_farthest(w_groups, alpha):
    """Planted: the beta-step takes the farthest code."""
    a = np.asarray(alpha, dtype=np.float64)
    S = O._code_signs(a.shape[0])
    vals = np.einsum("cq,q...->...c", S, a)
    d = np.abs(np.asarray(w_groups)[..., :, None] - vals[..., None, :])
    return np.moveaxis(S[np.argmax(d, axis=-1)], -1, 0)


def _nearest_bits_reversed(w_groups, alpha):
    """Planted: code bit i mapped to plane q-1-i."""
    return O.nearest_codes(w_groups, np.asarray(alpha)[::-1])


@pytest.mark.parametrize("mutant", [_fit_no_residual, _fit_alpha_not_rounded_for_signs])
def test_fit_pins_catch_mistakes(mutant):
    assert not (pin_fit_q1_closed_form(mutant) and pin_fit_exact_recovery(mutant)
                and pin_fit_q1_global_optimum(mutant) and pin_fit_stored_signs_are_best(mutant))


@pytest.mark.parametrize("mutant", [_nearest_farthest, _nearest_bits_reversed])
def test_nearest_codes_pin_catches_mistakes(mutant):
    assert not pin_nearest_codes_bruteforce(mutant)


# ---------------------------------------------------------------------------
# Variable-grid fitting (planes + one constant per group): at q = 1 it is
# Lloyd's two-level algorithm (checked against scikit-learn's k-means),
# representable grids are recovered exactly, stored points are the nearest
# grid points by brute force, the error never rises, and planted mistakes fail.
# ---------------------------------------------------------------------------
def pin_grid_q1_is_lloyd(fit_groups) -> bool:
    """q = 1: the two grid points off -/+ alpha after k rounds are the centres
    k-means (Lloyd, two clusters) reaches in k iterations from the greedy start."""
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(21)
    w = (rng.standard_normal((3, 128)) * 0.02 + rng.standard_normal((3, 1)) * 0.01).astype(np.float16)
    g = 64
    for iters in (1, 3):
        _, a0, off0, _ = fit_groups(w, 1, g, 0)
        _, a, off, _ = fit_groups(w, 1, g, iters)
        for j in range(3):
            for G in range(2):
                x = w[j, G * g:(G + 1) * g].astype(np.float64)[:, None]
                init = np.array([[off0[j, G] - a0[0, j, G]], [off0[j, G] + a0[0, j, G]]])
                km = KMeans(n_clusters=2, init=init, n_init=1, max_iter=iters, tol=0.0, algorithm="lloyd").fit(x)
                want = np.sort(km.cluster_centers_[:, 0])
                got = np.sort([off[j, G] - a[0, j, G], off[j, G] + a[0, j, G]])
                if not np.allclose(got, want, rtol=0, atol=1e-12):
                    return False
    return True


def pin_grid_exact_recovery(fit) -> bool:
    """w = off + c (b1 + b2 / 2): signs, scales, offset recovered, error 0."""
    rng = np.random.default_rng(22)
    m, ng, g = 4, 3, 128
    c = 2.0 ** rng.integers(-9, -5, size=(m, ng))
    off = rng.integers(-64, 64, size=(m, ng)) * 2.0 ** -12
    b = rng.choice([-1.0, 1.0], size=(2, m, ng, g))
    w = (off[..., None] + c[..., None] * (b[0] + b[1] / 2)).reshape(m, ng * g).astype(np.float16)
    signs, alpha, offset, err = fit(w, 2, g, 3)
    return (np.array_equal(signs.reshape(2, m, ng, g), b.astype(np.int8))
            and np.array_equal(alpha.astype(np.float64), np.stack([c, c / 2]).transpose(0, 2, 1))
            and np.array_equal(offset.astype(np.float64), off.T) and float(np.abs(err).max()) == 0.0)


def pin_grid_stored_points_are_nearest(fit) -> bool:
    rng = np.random.default_rng(23)
    q, g, m, n = 3, 64, 10, 256
    w = (rng.standard_normal((m, n)) * 0.02 + 0.015).astype(np.float16)
    signs, alpha, offset, err = fit(w, q, g, 2)
    combos = np.array(list(itertools.product([-1.0, 1.0], repeat=q)))
    for j in range(m):
        for G in range(n // g):
            a = alpha[:, G, j].astype(np.float64)
            o = float(offset[G, j])
            vals = o + combos @ a
            wk = w[j, G * g:(G + 1) * g].astype(np.float64)
            v = o + np.einsum("i,ik->k", a, signs[:, j, G * g:(G + 1) * g].astype(np.float64))
            best = np.abs(wk[:, None] - vals[None, :]).min(axis=1)
            if np.any(np.abs(wk - v) > best + 1e-15):
                return False
            e = float(((wk - v) ** 2).sum())
            if abs(e - err[G, j]) > 1e-12 * max(e, 1e-30):
                return False
    return True


def test_grid_pins():
    assert pin_grid_q1_is_lloyd(O._fit_groups_grid)
    assert pin_grid_exact_recovery(O.fit_bcq_grid)
    assert pin_grid_stored_points_are_nearest(O.fit_bcq_grid)


@pytest.mark.parametrize("q,g", [(1, 64), (2, 64), (3, 128), (4, 128)])
def test_grid_error_never_rises_and_beats_plain_bcq_on_shifted_weights(q, g):
    rng = np.random.default_rng(24 + q)
    w = (rng.standard_normal((6, 512)) * 0.02 + 0.02).astype(np.float16)
    trace = O.fit_bcq_grid_trace(w, q, g, 4)
    scale = (w.astype(np.float64).reshape(6, -1, g) ** 2).sum(-1)
    for before, after in zip(trace, trace[1:]):
        assert np.all(after <= before + 1e-12 * scale)
    # The plain BCQ grid is symmetric about 0; a constant per group can only help.
    assert O.fit_bcq_grid(w, q, g, 4)[3].sum() < O.fit_bcq(w, q, g, 4)[2].sum()


def test_grid_step_matches_least_squares():
    rng = np.random.default_rng(25)
    q, g = 3, 64
    B = rng.choice([-1.0, 1.0], size=(q, 7, g))
    w = rng.standard_normal((7, g)) + 0.5
    a, off = O._ls_grid(w, B, np.zeros((q, 7)), np.zeros(7), g)
    for r in range(7):
        X = np.concatenate([B[:, r, :].T, np.ones((g, 1))], axis=1)
        ref = np.linalg.lstsq(X, w[r], rcond=None)[0]
        assert np.allclose(np.append(a[:, r], off[r]), ref, rtol=1e-10, atol=1e-12)


def test_grid_step_keeps_values_when_a_plane_is_constant():
    rng = np.random.default_rng(26)
    B = rng.choice([-1.0, 1.0], size=(2, 1, 32))
    B[1] = 1.0                                      # plane 1 = the ones column: singular
    a_old, off_old = np.array([[0.3], [0.2]]), np.array([0.05])
    a, off = O._ls_grid(rng.standard_normal((1, 32)), B, a_old, off_old, 32)
    assert np.array_equal(a, a_old) and np.array_equal(off, off_old)


def _grid_groups_offset_frozen(w, q, g, iters, trace=None):
    """Planted: the offset stays at the group mean (only the scales are refit)."""
    W = np.asarray(w, dtype=np.float64)
    m, n = W.shape
    Wg = W.reshape(m, n // g, g)
    off = Wg.mean(-1)
    r = Wg - off[..., None]
    B = np.empty((q,) + Wg.shape)
    a = np.empty((q,) + Wg.shape[:-1])
    for i in range(q):
        B[i] = np.where(r >= 0, 1.0, -1.0)
        a[i] = (B[i] * r).sum(-1) / g
        r -= a[i][..., None] * B[i]
    for _ in range(iters):
        a = O._ls_alpha(Wg - off[..., None], B, a, g)
        B = O.nearest_grid_codes(Wg, a, off)
    return Wg, a, off, B


def _grid_fit_offset_ignored_in_codes(w, q, g, iters):
    """Planted: the last nearest-point step forgets the offset."""
    Wg, a, off, _ = O._fit_groups_grid(w, q, g, iters)
    a16, off32 = a.astype(np.float16), off.astype(np.float32)
    B = O.nearest_codes(Wg, a16.astype(np.float64))
    err = ((Wg - O._grid_value(a16.astype(np.float64), off32.astype(np.float64), B)) ** 2).sum(-1)
    m, ng, _ = Wg.shape
    return B.reshape(q, m, ng * g).astype(np.int8), np.transpose(a16, (0, 2, 1)), off32.T, err.T


def _grid_fit_offset_negated(w, q, g, iters):
    """Planted: the stored offset has the wrong sign."""
    s, a, off, err = O.fit_bcq_grid(w, q, g, iters)
    return s, a, -off, err


def test_grid_pins_catch_mistakes():
    assert not pin_grid_q1_is_lloyd(_grid_groups_offset_frozen)
    for mutant in (_grid_fit_offset_ignored_in_codes, _grid_fit_offset_negated):
        assert not (pin_grid_exact_recovery(mutant) and pin_grid_stored_points_are_nearest(mutant))
