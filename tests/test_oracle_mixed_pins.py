"""Pins of the oracle's mixed 2/4/16-bit format (CPU only).

The format (precision blocks of 32 rows x 1024 inputs with their own plane
count, plus sparse fp16 outliers added to the BCQ value) is this library's
reading of the OpenAlex record "Fast and Efficient 2-bit LLM Inference on GPU:
2/4/16-bit in a Weight Matrix with Asynchronous Dequantization" (abstract).
The oracle is pinned here against hand-derived values (tests/golden), brute
force, the plain BCQ oracle it reduces to, and scipy's sparse product; planted
mistakes must fail at least one pin.
"""
from __future__ import annotations

import json
import os

import numpy as np
import pytest

from oracle import bcq_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden", "mixed_format.json")


def _gold():
    with open(GOLD) as f:
        return json.load(f)


def _layout_signs(case):
    s = -np.ones((case["q_max"], case["m"], case["n"]), dtype=np.int8)
    for i, r, k in case["plus_one"]:
        s[i, r, k] = 1
    return s


def pin_layout_golden(pack_mixed, offsets) -> bool:
    c = _gold()["layout_case"]
    bp = np.array(c["block_planes"], dtype=np.uint8)
    if not np.array_equal(np.asarray(offsets(bp)), np.array(c["offsets"])):
        return False
    want = np.zeros(c["total_bytes"], dtype=np.uint8)
    for off, v in c["nonzero"].items():
        want[int(off)] = v
    return np.array_equal(np.asarray(pack_mixed(_layout_signs(c), bp)), want)


def pin_pairs_golden(pack_mixed) -> bool:
    """Blocks of three and four planes: the planes are stored in pairs."""
    for c in _gold()["pairs_cases"]:
        bp = np.array(c["block_planes"], dtype=np.uint8)
        want = np.zeros(c["total_bytes"], dtype=np.uint8)
        for off, v in c["nonzero"].items():
            want[int(off)] = v
        if not np.array_equal(np.asarray(pack_mixed(_layout_signs(c), bp)), want):
            return False
    return True


def pin_unpack_golden(unpack_mixed) -> bool:
    c = _gold()["layout_case"]
    bp = np.array(c["block_planes"], dtype=np.uint8)
    buf = np.zeros(c["total_bytes"], dtype=np.uint8)
    for off, v in c["nonzero"].items():
        buf[int(off)] = v
    got = np.asarray(unpack_mixed(buf, bp, c["q_max"], c["m"], c["n"]))
    want = _layout_signs(c)
    # Planes a block does not store come back as 0.
    for s_ in range(bp.shape[0]):
        for R in range(bp.shape[1]):
            want[bp[s_, R]:, 32 * R: 32 * R + 32, 1024 * s_: 1024 * s_ + 1024] = 0
    return np.array_equal(got, want)


def _values_inputs(c):
    q, m, n, g = c["q_max"], c["m"], c["n"], c["g"]
    signs = np.empty((q, m, n), dtype=np.int8)
    signs[0], signs[1] = c["plane0_sign"], c["plane1_sign"]
    alpha = np.empty((q, n // g, m), dtype=np.float16)
    for G in range(n // g):
        alpha[0, G, :] = c["alpha"]["plane0"][G]
        alpha[1, G, :] = c["alpha"]["plane1"][G]
    rows = sorted(c["outliers"]["row_ptr_rows"])
    row_ptr = np.zeros(m + 1, dtype=np.int64)
    for r, _, _ in rows:
        row_ptr[r + 1:] += 1
    col = np.array([k for _, k, _ in rows])
    val = np.array([v for _, _, v in rows], dtype=np.float16)
    return signs, alpha, np.array(c["block_planes"], dtype=np.uint8), (row_ptr, col, val)


def pin_values_golden(weights, matmul) -> bool:
    c = _gold()["values_case"]
    signs, alpha, bp, outl = _values_inputs(c)
    W = np.asarray(weights(signs, alpha, bp, c["g"], outl))
    if not all(W[r, k] == v for r, k, v in c["weights"]):
        return False
    y = np.asarray(matmul(np.ones((1, c["n"])), signs, alpha, bp, c["g"], outl))
    return all(y[0, r] == v for r, v in c["y_for_ones"])


def pin_outlier_layout_golden(pack_outliers) -> bool:
    c = _gold()["outlier_layout_case"]
    optr, oent = pack_outliers(np.array(c["row_ptr"]), np.array(c["col"]),
                               np.array(c["val"], dtype=np.float16), c["m"], c["n"])
    return np.array_equal(np.asarray(optr), c["optr"]) and np.array_equal(np.asarray(oent), c["oent"])


def _brute_y(x, signs, alpha, bp, g, outl):
    x = np.asarray(x, dtype=np.float64)
    q, m, n = signs.shape
    rp, col, val = outl
    y = np.zeros((x.shape[0], m))
    for b in range(x.shape[0]):
        for j in range(m):
            acc = 0.0
            for k in range(n):
                qb = int(bp[k // 1024, j // 32])
                for i in range(qb):
                    acc += float(alpha[i, k // g, j]) * float(signs[i, j, k]) * x[b, k]
            for e in range(rp[j], rp[j + 1]):
                acc += float(val[e]) * x[b, col[e]]
            y[b, j] = acc
    return y


def _random_mixed(seed, q, m, n, g, density=0.01):
    rng = np.random.default_rng(seed)
    signs = rng.choice(np.array([-1, 1], dtype=np.int8), size=(q, m, n))
    alpha = np.abs(rng.normal(0, 0.02, (q, n // g, m))).astype(np.float16)
    bp = rng.integers(1, q + 1, (-(-n // 1024), -(-m // 32))).astype(np.uint8)
    nnz = max(1, int(density * m * n))
    flat = np.sort(rng.choice(m * n, nnz, replace=False))
    rows, cols = flat // n, flat % n
    row_ptr = np.concatenate([[0], np.cumsum(np.bincount(rows, minlength=m))])
    val = rng.normal(0, 0.1, nnz).astype(np.float16)
    x = rng.normal(0, 1, (2, n)).astype(np.float16)
    return signs, alpha, bp, (row_ptr, cols, val), x


def pin_bruteforce(matmul) -> bool:
    signs, alpha, bp, outl, x = _random_mixed(1, 3, 40, 2100, 84)
    y = np.asarray(matmul(x, signs, alpha, bp, 84, outl))
    want = _brute_y(x, signs, alpha, bp, 84, outl)
    return bool(np.all(np.abs(y - want) <= 1e-12 * (np.abs(want) + 1.0)))


def _distinct(q, ng, m):
    return np.arange(1, q * ng * m + 1, dtype=np.uint16).reshape(q, ng, m).view(np.float16)


def pin_mixed_scales_golden(pack) -> bool:
    for c in _gold()["scales_cases"]:
        a = _distinct(c["q_max"], c["n"] // c["g"], c["m"])
        out = np.asarray(pack(a, np.array(c["block_planes"], dtype=np.uint8), c["g"]), dtype=np.float16)
        if out.size != c["nelem"]:
            return False
        bits = out.view(np.uint16)
        for e in c["entries"]:
            want = 0 if e[1] is None else int(a.view(np.uint16)[e[1], e[2], e[3]])
            if int(bits[e[0]]) != want:
                return False
    return True


# ---------------------------------------------------------------------------
# The pins on the real oracle.
# ---------------------------------------------------------------------------
def test_mixed_layout_pins():
    assert pin_layout_golden(O.pack_mixed, O.mixed_block_offsets)
    assert pin_pairs_golden(O.pack_mixed)
    assert pin_unpack_golden(O.unpack_mixed)
    for c in _gold()["pairs_cases"]:
        bp = np.array(c["block_planes"], dtype=np.uint8)
        buf = np.zeros(c["total_bytes"], dtype=np.uint8)
        for off, v in c["nonzero"].items():
            buf[int(off)] = v
        assert np.array_equal(O.unpack_mixed(buf, bp, c["q_max"], c["m"], c["n"]), _layout_signs(c))


def test_mixed_value_pins():
    assert pin_values_golden(O.mixed_weights, O.mixed_matmul)
    assert pin_bruteforce(O.mixed_matmul)


def test_outlier_layout_pin():
    assert pin_outlier_layout_golden(O.pack_outliers)


@pytest.mark.parametrize("q,m,n,g", [(3, 45, 2056, 8), (2, 70, 3000, 40), (4, 33, 1032, 8)])
def test_equal_plane_counts_reduce_to_plain_bcq(q, m, n, g):
    """Every block at q planes and no outliers: the product is bcq_matmul's,
    and with at most two planes the buffer is pack_bcq's."""
    signs, alpha, _, _, x = _random_mixed(q + m, q, m, n, g)
    bp = np.full((-(-n // 1024), -(-m // 32)), q, dtype=np.uint8)
    assert np.array_equal(O.mixed_matmul(x, signs, alpha, bp, g), O.bcq_matmul(x, signs, alpha, g))
    s2 = signs[:2]
    bp2 = np.full_like(bp, 2)
    assert np.array_equal(O.pack_mixed(s2, bp2), O.pack_bcq(s2))


def test_outliers_alone_are_the_sparse_product():
    """With every scale 0 the product is S x, checked with scipy's CSR product."""
    import scipy.sparse as sp
    signs, alpha, bp, (rp, col, val), x = _random_mixed(9, 2, 70, 3000, 40, density=0.02)
    y = O.mixed_matmul(x, signs, np.zeros_like(alpha), bp, 40, (rp, col, val))
    S_ = sp.csr_matrix((val.astype(np.float64), col, rp), shape=(70, 3000))
    want = (S_ @ x.astype(np.float64).T).T
    assert np.allclose(y, want, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("q,m,n", [(4, 70, 3000), (2, 33, 1032), (3, 64, 2048)])
def test_mixed_roundtrips(q, m, n):
    signs, _, bp, (rp, col, val), _ = _random_mixed(q * m, q, m, n, 8)
    pk = O.pack_mixed(signs, bp)
    assert pk.size == O.mixed_packed_nbytes(bp) == int(O.mixed_block_offsets(bp)[-1]) * 4096
    got = O.unpack_mixed(pk, bp, q, m, n)
    qb = np.repeat(np.repeat(bp.T, 32, axis=0)[:m], 1024, axis=1)[:, :n]
    for i in range(q):
        present = i < qb
        assert np.array_equal(got[i][present], signs[i][present])
        assert not got[i][~present].any()
    optr, oent = O.pack_outliers(rp, col, val, m, n)
    assert np.array_equal(O.unpack_outliers(optr, oent, m, n), O.outlier_dense(rp, col, val, m, n))


@pytest.mark.parametrize("tiles", [[0], [1, 3], [0, 2, 3]])
def test_tile_rows_equal_the_whole_product(tiles):
    signs, alpha, bp, outl, x = _random_mixed(21, 4, 100, 2100, 84)
    pk = O.pack_mixed(signs, bp)
    y, rows = O.mixed_matmul_tiles(x, pk, bp, alpha, 84, 100, 2100, tiles, outl)
    full = O.mixed_matmul(x, signs, alpha, bp, 84, outl)
    assert np.array_equal(rows, np.concatenate([np.arange(32 * t, min(100, 32 * t + 32)) for t in tiles]))
    assert np.allclose(y, full[:, rows], rtol=1e-13, atol=1e-13)


def test_mixed_scales_pins():
    assert pin_mixed_scales_golden(O.pack_mixed_scales)


@pytest.mark.parametrize("q,m,n,g", [(2, 40, 2048, 64), (1, 33, 1152, 128), (2, 64, 3072, 256)])
def test_mixed_scales_reduce_to_unit_major_scales(q, m, n, g):
    """Every block at q <= 2 planes: the buffer is pack_scales's."""
    a = _distinct(q, n // g, m)
    bp = np.full((-(-n // 1024), -(-m // 32)), q, dtype=np.uint8)
    assert np.array_equal(O.pack_mixed_scales(a, bp, g).view(np.uint16), O.pack_scales(a, g).view(np.uint16))


@pytest.mark.parametrize("q_max,m,n,g", [(4, 70, 3072, 64), (3, 33, 2048, 128), (4, 64, 2048, 256)])
def test_mixed_scales_roundtrip(q_max, m, n, g):
    rng = np.random.default_rng(q_max + m)
    bp = rng.integers(1, q_max + 1, (-(-n // 1024), -(-m // 32))).astype(np.uint8)
    a = _distinct(q_max, n // g, m)
    buf = O.pack_mixed_scales(a, bp, g)
    assert buf.size * 2 == O.mixed_scales_nbytes(bp, g)
    back = O.unpack_mixed_scales(buf, bp, q_max, m, n, g)
    # Each (plane, group, row) comes back where its block stores the plane, else 0.
    for s_ in range(bp.shape[0]):
        for R in range(bp.shape[1]):
            rows = slice(32 * R, min(m, 32 * R + 32))
            groups = sorted({k // g for k in range(1024 * s_, min(n, 1024 * s_ + 1024))})
            for G in groups:
                qb = int(bp[s_, R])
                assert np.array_equal(back[:qb, G, rows].view(np.uint16), a[:qb, G, rows].view(np.uint16))


def _mixed_scales_pairs_swapped(alpha, bp, g):
    # Pair 1 of each 3- or 4-plane block stored before pair 0.
    out = O.pack_mixed_scales(alpha, bp, g).copy()
    H = 2 if g == 64 else 1
    off = O.mixed_block_offsets(bp)
    for u, qb in enumerate(np.asarray(bp).reshape(-1)):
        if qb >= 3:
            base = int(off[u]) * 256 * H
            p0 = out[base: base + 512 * H].copy()
            e1 = int(qb) - 2
            p1 = out[base + 512 * H: base + 512 * H + 256 * H * e1].copy()
            out[base: base + p1.size] = p1
            out[base + p1.size: base + p1.size + p0.size] = p0
    return out


def test_mixed_scales_pins_catch_mistakes():
    assert not pin_mixed_scales_golden(_mixed_scales_pairs_swapped)


def test_mixed_rejects_bad_inputs():
    signs, alpha, bp, outl, _ = _random_mixed(3, 2, 40, 2048, 64)
    with pytest.raises(ValueError):
        O.pack_mixed(signs, np.full_like(bp, 3))          # more planes than given
    with pytest.raises(ValueError):
        O.pack_mixed(signs, np.zeros_like(bp))            # a block with no plane
    rp, col, val = outl
    bad = col.copy()
    if rp[1] - rp[0] >= 2:
        bad[rp[0]], bad[rp[0] + 1] = bad[rp[0] + 1], bad[rp[0]]
    else:
        bad[0] = 5000
    with pytest.raises(ValueError):
        O.outlier_dense(rp, bad, val, 40, 2048)


# ---------------------------------------------------------------------------
# Planted mistakes: each must make at least one pin fail.
# ---------------------------------------------------------------------------
def _w_outlier_replaces(signs, alpha, bp, g, outl=None):
    W = O.mixed_weights(signs, alpha, bp, g, None)
    if outl is not None:
        S_ = O.outlier_dense(*outl, W.shape[0], W.shape[1])
        W = np.where(S_ != 0, S_, W)
    return W


def _w_all_planes(signs, alpha, bp, g, outl=None):
    q = signs.shape[0]
    return O.mixed_weights(signs, alpha, np.full_like(np.asarray(bp), q), g, outl)


def _w_block_by_group(signs, alpha, bp, g, outl=None):
    # Plane count looked up by the scale group instead of the 1024-input slice.
    q, m, n = signs.shape
    W = np.zeros((m, n))
    a = np.asarray(alpha, dtype=np.float64)
    for j in range(m):
        for k in range(n):
            qb = int(np.asarray(bp)[min(k // g, np.asarray(bp).shape[0] - 1), j // 32])
            W[j, k] = sum(a[i, k // g, j] * signs[i, j, k] for i in range(qb))
    if outl is not None:
        W += O.outlier_dense(*outl, m, n)
    return W


def _mm(wfn):
    return lambda x, s, a, bp, g, outl=None: np.asarray(x, dtype=np.float64) @ wfn(s, a, bp, g, outl).T


@pytest.mark.parametrize("wfn", [_w_outlier_replaces, _w_all_planes, _w_block_by_group])
def test_value_pins_catch_mistakes(wfn):
    assert not (pin_values_golden(wfn, _mm(wfn)) and pin_bruteforce(_mm(wfn)))


def _offsets_inclusive(bp):
    return np.cumsum(np.asarray(bp, dtype=np.int64).reshape(-1)).astype(np.uint32)


def _pack_plane_major(signs, bp):
    # Planes outermost inside a block: chunk (i, U) at (i*8 + U)*512.
    out = []
    bp = np.asarray(bp)
    for s_ in range(bp.shape[0]):
        for R in range(bp.shape[1]):
            qb = int(bp[s_, R])
            blk = O.pack_bcq(signs[:qb, 32 * R: 32 * R + 32, 1024 * s_: 1024 * s_ + 1024]).reshape(8, qb, 512)
            out.append(blk.transpose(1, 0, 2).reshape(-1))
    return np.concatenate(out)


def _pack_unpaired(signs, bp):
    # All of a block's planes in one chunk sequence: chunk (U, i) at (U*q_b + i)*512.
    out = []
    bp = np.asarray(bp)
    for s_ in range(bp.shape[0]):
        for R in range(bp.shape[1]):
            qb = int(bp[s_, R])
            out.append(O.pack_bcq(signs[:qb, 32 * R: 32 * R + 32, 1024 * s_: 1024 * s_ + 1024]))
    return np.concatenate(out)


def test_layout_pins_catch_mistakes():
    assert not pin_layout_golden(O.pack_mixed, _offsets_inclusive)
    assert not (pin_layout_golden(_pack_plane_major, O.mixed_block_offsets) and pin_pairs_golden(_pack_plane_major))
    assert not pin_pairs_golden(_pack_unpaired)


def _outliers_absolute_k(rp, col, val, m, n):
    optr, oent = O.pack_outliers(rp, col, val, m, n)
    # Entries keep the absolute input index instead of the index in the slice.
    c = np.asarray(col)
    fixed = [(int(e) & 0xFFFF0000) | int(k) for e, k in zip(oent, [c[i] for i in range(len(c))])]
    return optr, np.asarray(fixed, dtype=np.uint32)


def _outliers_row_major(rp, col, val, m, n):
    bits = np.asarray(val, dtype=np.float16).view(np.uint16).astype(np.uint32)
    c = np.asarray(col, dtype=np.int64)
    return np.asarray(rp, dtype=np.uint32), ((c % 1024) | (bits << 16)).astype(np.uint32)


@pytest.mark.parametrize("fn", [_outliers_absolute_k, _outliers_row_major])
def test_outlier_pin_catches_mistakes(fn):
    assert not pin_outlier_layout_golden(fn)
