"""FP64 CPU oracle for LUT-GEMM over binary-coding-quantised (BCQ) weights.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import or call this module.  The product
path (the CUDA library and its Python binding) never imports it, and this
module imports nothing from the product: the two share no code.  Inputs come
from ``bcq_synth`` (random draws only).

What it computes, and where the pages say so
--------------------------------------------
Source pages: "LUT-GEMM -- paper by Park et al. (2022), ICLR 2024" (Elamur
card; sections *Summary*, *Interesting ideas*) and the pith.science card of the
same paper (abstract).

* BCQ format (Summary; Interesting ideas, "Lookup tables instead of
  multiplications"): a weight row is a sum of q binary {-1,+1} vectors, each
  with a scale.  Scales are group-wise (Summary; "Group size as a separate
  hyper-parameter"): W[j,k] = sum_i alpha[i, k//g, j] * beta[i, j, k].
* Uniform quantisation is a special case of BCQ (Summary; "One format for many
  schemes").  The pages give no formula; the closed form used here is derived in
  ``uniform_to_bcq``.  It needs a per-group offset term (off[k//g, j]).
* The product y = W x is what LUT-GEMM returns "with no dequantization"
  (Summary): the lookup form is an exact regrouping of this sum, so the oracle's
  reference result is the plain dequantise-then-matmul in FP64
  (``bcq_matmul``).  ``lut_matmul`` writes the lookup regrouping out plainly so
  the identity itself can be pinned.
* Lookup table (Interesting ideas): for a run of mu = 8 activations, the 256
  possible signed sums are computed once; T[p] = sum_t (2*bit_t(p) - 1) * x_t.

Readings where the pages are silent (each also listed in the design notes):

* bit t of a table index / packed byte stands for activation 8c + t (LSB
  first); bit value 1 means beta = +1.
* plane i (0-based) of a converted uniform weight is bit i of the integer code.
* the packed weight layout is this library's own tiled layout; it is defined
  in ``include/lutgemm.h`` and re-implemented here from that text
  (``pack_bcq`` / ``unpack_bcq``).  So is the unit-major scale layout
  (``pack_scales`` / ``unpack_scales``).

Parity status: every public function here is pinned by
``tests/test_oracle_pins.py`` against brute force, closed forms, special cases
or hand-derived fixtures (tests/golden).  None is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

MU = 8            # activations per lookup-table run (256-entry tables)
SLICE = 1024      # inputs per slice of the packed layout
TILE_ROWS = 32    # rows per row tile of the packed layout
PIECE = 128       # inputs per 16-byte lane piece of the packed layout
BLOCK_BYTES = 4096  # bytes of one (slice, row tile, plane): 8 chunks of 512

__all__ = [
    "lut_table", "dequantize_bcq", "bcq_matmul", "lut_matmul",
    "packed_nbytes", "pack_bcq", "unpack_bcq", "unpack_rows", "unpack_bcq_vec", "packed_row_tiles",
    "scales_nbytes", "pack_scales", "unpack_scales",
    "uniform_to_bcq", "uniform_dequant", "bcq_matmul_rows",
    "fit_bcq", "fit_bcq_trace", "nearest_codes",
    "fit_bcq_grid", "fit_bcq_grid_trace", "nearest_grid_codes",
    "mixed_block_offsets", "mixed_packed_nbytes", "pack_mixed", "unpack_mixed",
    "mixed_weights", "mixed_matmul", "pack_outliers", "unpack_outliers", "outlier_dense",
    "mixed_matmul_tiles", "mixed_scales_nbytes", "pack_mixed_scales", "unpack_mixed_scales",
]


# ---------------------------------------------------------------------------
# Lookup table (Interesting ideas: "the possible sums of activation
# sub-vectors can be computed once and then simply looked up").
# ---------------------------------------------------------------------------
def lut_table(xchunk) -> np.ndarray:
    """All 256 signed sums of one run of 8 activations, in FP64.

    T[p] = sum_{t=0..7} (2*bit_t(p) - 1) * x[t], bit t of p being (p >> t) & 1.
    """
    x = np.asarray(xchunk, dtype=np.float64).reshape(MU)
    p = np.arange(256)
    bits = (p[:, None] >> np.arange(MU)[None, :]) & 1          # [256, 8]
    signs = 2.0 * bits.astype(np.float64) - 1.0
    return signs @ x


# ---------------------------------------------------------------------------
# BCQ dequantisation and the plain product (Summary; Interesting ideas).
# ---------------------------------------------------------------------------
def dequantize_bcq(signs, alpha, g: int, offset=None) -> np.ndarray:
    """W[j,k] = sum_i alpha[i, k//g, j] * signs[i, j, k] (+ offset[k//g, j]), FP64 [m][n].

    signs: [q][m][n] of -1/+1; alpha: [q][n/g][m] (fp16 or wider);
    offset: [n/g][m] or None (pure BCQ).
    """
    s = np.asarray(signs)
    q, m, n = s.shape
    a = np.asarray(alpha, dtype=np.float64)
    assert a.shape == (q, n // g, m), (a.shape, (q, n // g, m))
    W = np.zeros((m, n), dtype=np.float64)
    for i in range(q):
        a_rows = np.repeat(a[i], g, axis=0).T          # [m][n]: alpha of (row, input)
        W += a_rows * s[i].astype(np.float64)
    if offset is not None:
        o = np.asarray(offset, dtype=np.float64)
        assert o.shape == (n // g, m)
        W += np.repeat(o, g, axis=0).T
    return W


def bcq_matmul(x, signs, alpha, g: int, offset=None) -> np.ndarray:
    """y[b, j] = sum_k W[j, k] * x[b, k] with W from ``dequantize_bcq``; FP64 [batch][m]."""
    W = dequantize_bcq(signs, alpha, g, offset)
    xx = np.asarray(x, dtype=np.float64)
    return xx @ W.T


def bcq_matmul_rows(x, signs_rows, alpha_rows, g: int, offset_rows=None) -> np.ndarray:
    """``bcq_matmul`` restricted to a subset of output rows.

    signs_rows: [q][r][n]; alpha_rows: [q][n/g][r]; offset_rows: [n/g][r] or None.
    Returns [batch][r].  Used to check sampled outputs of large problems.
    """
    return bcq_matmul(x, signs_rows, alpha_rows, g, offset_rows)


def lut_matmul(x, signs, alpha, g: int, offset=None) -> np.ndarray:
    """The lookup-table regrouping of ``bcq_matmul``, written out plainly (FP64).

    For every batch column b and run c of 8 inputs, the 256-entry table
    T = lut_table(x[b, 8c:8c+8]) is built once; each plane-row then reads one
    entry, indexed by the byte of its 8 sign bits (bit t = 1 iff sign = +1),
    and scales it by the alpha of the run's group.  The offset of a converted
    uniform weight multiplies the group's activation sum.  Requires g % 8 == 0.
    """
    s = np.asarray(signs)
    q, m, n = s.shape
    assert n % MU == 0 and g % MU == 0 and n % g == 0
    a = np.asarray(alpha, dtype=np.float64)
    xx = np.asarray(x, dtype=np.float64)
    batch = xx.shape[0]
    weights = (1 << np.arange(MU)).astype(np.int64)
    y = np.zeros((batch, m), dtype=np.float64)
    for b in range(batch):
        for c in range(n // MU):
            T = lut_table(xx[b, MU * c: MU * c + MU])
            G = (MU * c) // g
            for i in range(q):
                bits = (s[i, :, MU * c: MU * c + MU] > 0).astype(np.int64)   # [m][8]
                idx = bits @ weights                                           # [m]
                y[b] += a[i, G, :] * T[idx]
        if offset is not None:
            o = np.asarray(offset, dtype=np.float64)
            for G in range(n // g):
                y[b] += o[G, :] * xx[b, G * g:(G + 1) * g].sum()
    return y


# ---------------------------------------------------------------------------
# Packed layout (library-defined; re-implemented from the header's text).
#
#   n_s = ceil(n / 1024) slices, m_t = ceil(m / 32) row tiles.
#   The buffer is n_s * m_t * 8 * q chunks of 512 bytes; chunk (s, R, U, i)
#   starts at byte (((s * m_t + R) * 8 + U) * q + i) * 512.
#   In that chunk, byte l*16 + j (l < 32, j < 16) holds the 8 sign bits of
#   row r = 32*R + l, plane i, inputs k = 1024*s + 128*P + 8*c + t (bit t,
#   LSB first), where P = U xor (4 * (l // 16)) and c = j xor (l % 16).
#   A bit is 1 iff the sign is +1; bits of rows >= m or inputs >= n are 0.
# ---------------------------------------------------------------------------
def packed_nbytes(q: int, m: int, n: int) -> int:
    return math.ceil(n / SLICE) * math.ceil(m / TILE_ROWS) * q * BLOCK_BYTES


def _piece_and_run(U: int, l: int, j: int):
    """(P, c): which 128-input piece and which 8-input run byte (U, l, j) holds."""
    return U ^ (4 * (l // 16)), j ^ (l % 16)


def pack_bcq(signs) -> np.ndarray:
    """int8 signs [q][m][n] (-1/+1) -> packed uint8 buffer of ``packed_nbytes`` bytes."""
    s = np.asarray(signs)
    q, m, n = s.shape
    if not np.all((s == 1) | (s == -1)):
        raise ValueError("signs must be -1 or +1")
    ns, mt = math.ceil(n / SLICE), math.ceil(m / TILE_ROWS)
    bits = np.zeros((q, mt * TILE_ROWS, ns * SLICE), dtype=np.uint8)
    bits[:, :m, :n] = (s > 0)
    # bits_r[i, R, l, s, k_in_slice]
    bits_r = bits.reshape(q, mt, TILE_ROWS, ns, SLICE)
    out = np.zeros((ns, mt, 8, q, TILE_ROWS, 16), dtype=np.uint8)
    for U in range(8):
        for l in range(TILE_ROWS):
            for j in range(16):
                P, c = _piece_and_run(U, l, j)
                k0 = PIECE * P + MU * c
                byte = np.zeros((q, mt, ns), dtype=np.uint8)
                for t in range(MU):
                    byte |= (bits_r[:, :, l, :, k0 + t] << t).astype(np.uint8)
                out[:, :, U, :, l, j] = byte.transpose(2, 1, 0)
    return out.reshape(-1)


def unpack_bcq(packed, q: int, m: int, n: int) -> np.ndarray:
    """Inverse of ``pack_bcq``: packed bytes -> int8 signs [q][m][n]."""
    return unpack_rows(packed, q, m, n, np.arange(m))


def unpack_rows(packed, q: int, m: int, n: int, rows) -> np.ndarray:
    """Signs [q][len(rows)][n] of the given output rows, read from a packed buffer."""
    pk = np.asarray(packed, dtype=np.uint8).reshape(-1)
    assert pk.size == packed_nbytes(q, m, n)
    ns, mt = math.ceil(n / SLICE), math.ceil(m / TILE_ROWS)
    chunks = pk.reshape(ns, mt, 8, q, TILE_ROWS, 16)
    rows = np.asarray(rows, dtype=np.int64)
    out_bits = np.zeros((q, rows.size, ns * SLICE), dtype=np.uint8)
    for ri, r in enumerate(rows):
        R, l = divmod(int(r), TILE_ROWS)
        for U in range(8):
            for j in range(16):
                P, c = _piece_and_run(U, l, j)
                k0 = PIECE * P + MU * c
                byte = chunks[:, R, U, :, l, j]          # [ns][q]
                for t in range(MU):
                    bit = (byte >> t) & 1                 # [ns][q]
                    out_bits[:, ri, np.arange(ns) * SLICE + k0 + t] = bit.T
    bits = out_bits[:, :, :n]
    return (bits.astype(np.int8) * 2 - 1)


def unpack_bcq_vec(packed, q: int, m: int, n: int) -> np.ndarray:
    """``unpack_bcq`` with the layout's index map applied to whole arrays at
    once, for checking every output of full-size problems in seconds.

    Every byte is split into its 8 bits (bit t = input 8c + t, LSB first);
    then for each lane l the pieces and runs are put back in input order:
    piece P sits at step U = P xor 4*(l // 16) and run c at byte
    j = c xor (l % 16), the same map as ``unpack_rows``."""
    pk = np.asarray(packed, dtype=np.uint8).reshape(-1)
    assert pk.size == packed_nbytes(q, m, n)
    ns, mt = math.ceil(n / SLICE), math.ceil(m / TILE_ROWS)
    chunks = pk.reshape(ns, mt, 8, q, TILE_ROWS, 16)
    bits = np.unpackbits(chunks[..., None], axis=-1, bitorder="little")   # [ns][mt][U][q][l][j][t]
    out = np.empty((q, mt, TILE_ROWS, ns, SLICE), dtype=np.uint8)
    for l in range(TILE_ROWS):
        U_of_P = np.arange(8) ^ (4 * (l // 16))
        j_of_c = np.arange(16) ^ (l % 16)
        lane = bits[:, :, :, :, l][:, :, U_of_P][:, :, :, :, j_of_c]       # [ns][mt][P][q][c][t]
        out[:, :, l] = lane.transpose(3, 1, 0, 2, 4, 5).reshape(q, mt, ns, SLICE)
    out = out.reshape(q, mt * TILE_ROWS, ns * SLICE)
    return out[:, :m, :n].astype(np.int8) * 2 - 1


def packed_row_tiles(packed, q: int, m: int, n: int, R0: int, R1: int):
    """The bytes of row tiles [R0, R1) of a packed buffer, which are the packed
    buffer of the sub-matrix of rows 32*R0 .. min(m, 32*R1) - 1 (blocks are
    ordered slice-major, row tile minor).  Returns (buffer, rows of the sub-matrix)."""
    pk = np.asarray(packed, dtype=np.uint8).reshape(-1)
    assert pk.size == packed_nbytes(q, m, n)
    ns, mt = math.ceil(n / SLICE), math.ceil(m / TILE_ROWS)
    assert 0 <= R0 < R1 <= mt
    blocks = pk.reshape(ns, mt, q * BLOCK_BYTES)
    return np.ascontiguousarray(blocks[:, R0:R1]).reshape(-1), min(m, TILE_ROWS * R1) - TILE_ROWS * R0


# ---------------------------------------------------------------------------
# Unit-major scale layout (this library's own; defined in include/lutgemm.h).
# For g % 128 == 0 (one scale per 128-input piece, H = 1) and g == 64 (two,
# one per 64-input half of a piece, H = 2).  SP = min(q, 4), n_pg = ceil(q/4).
# Element (s, R, pg, l, U, e, h) sits at index
#   (((((s * m_t + R) * n_pg + pg) * 32 + l) * 8 + U) * SP + e) * H + h
# and holds alpha[4*pg + e][G][32*R + l], G = (1024*s + 128*P + 64*h) // g,
# P = U xor (4 * (l // 16)); 0 when the plane, row or piece half is out of
# range.
# ---------------------------------------------------------------------------
def _scale_dims(q: int, m: int, n: int, g: int):
    if not (g % PIECE == 0 or g == PIECE // 2) or n % g != 0:
        raise ValueError("the unit-major scale layout needs g % 128 == 0 or g == 64, and n % g == 0")
    return (math.ceil(n / SLICE), math.ceil(m / TILE_ROWS), min(q, 4), math.ceil(q / 4),
            2 if g == PIECE // 2 else 1)


def scales_nbytes(q: int, m: int, n: int, g: int) -> int:
    ns, mt, sp, npg, H = _scale_dims(q, m, n, g)
    return ns * mt * npg * 512 * sp * H


def pack_scales(alpha, g: int) -> np.ndarray:
    """fp16 alpha [q][n/g][m] -> fp16 unit-major scale buffer (1-D)."""
    a = np.asarray(alpha, dtype=np.float16)
    q, ng, m = a.shape
    n = ng * g
    ns, mt, sp, npg, H = _scale_dims(q, m, n, g)
    out = np.zeros((ns, mt, npg, TILE_ROWS, 8, sp, H), dtype=np.float16)
    for s_ in range(ns):
        for U in range(8):
            for half in range(2):                       # l // 16
                P = U ^ (4 * half)
                for h in range(H):
                    k0 = SLICE * s_ + PIECE * P + (PIECE // 2) * h
                    if k0 >= n:
                        continue                        # beyond n: stays 0
                    G = k0 // g
                    for pg in range(npg):
                        for e in range(sp):
                            i = 4 * pg + e
                            if i >= q:
                                continue                # padding plane: stays 0
                            col = np.zeros(mt * TILE_ROWS, dtype=np.float16)
                            col[:m] = a[i, G, :]
                            col = col.reshape(mt, TILE_ROWS)
                            lanes = slice(16 * half, 16 * half + 16)
                            out[s_, :, pg, lanes, U, e, h] = col[:, lanes]
    return out.reshape(-1)


def unpack_scales(scales, q: int, m: int, n: int, g: int) -> np.ndarray:
    """Inverse of ``pack_scales``: fp16 alpha [q][n/g][m] read back from the buffer.

    A group wider than one piece appears once per piece; every copy must agree.
    """
    ns, mt, sp, npg, H = _scale_dims(q, m, n, g)
    buf = np.asarray(scales, dtype=np.float16).reshape(ns, mt, npg, TILE_ROWS, 8, sp, H)
    ng = n // g
    out = np.full((q, ng, m), np.nan, dtype=np.float64)
    for s_ in range(ns):
        for U in range(8):
            for l in range(TILE_ROWS):
                P = U ^ (4 * (l // 16))
                for h in range(H):
                    k0 = SLICE * s_ + PIECE * P + (PIECE // 2) * h
                    if k0 >= n:
                        continue
                    G = k0 // g
                    rows = np.arange(mt) * TILE_ROWS + l
                    ok = rows < m
                    for i in range(q):
                        v = buf[s_, :, i // 4, l, U, i % 4, h].astype(np.float64)[ok]
                        prev = out[i, G, rows[ok]]
                        seen = ~np.isnan(prev)
                        if np.any(prev[seen] != v[seen]):
                            raise ValueError("copies of one group scale disagree")
                        out[i, G, rows[ok]] = v
    if np.isnan(out).any():
        raise ValueError("some scale never appears in the buffer")
    return out.astype(np.float16)


# ---------------------------------------------------------------------------
# Uniform quantisation rewritten as BCQ (Summary; Interesting ideas, "One
# format for many schemes").  The pages state that the rewrite exists but give
# no formula.  Derivation used here:
#   w = s * (c - z), c = sum_{i=0}^{q-1} 2^i * b_i with b_i in {0,1}.
#   With beta_i = 2*b_i - 1:  b_i = (beta_i + 1)/2, so
#   c = sum_i 2^(i-1) * beta_i + (2^q - 1)/2.
#   Hence w = sum_i (s * 2^(i-1)) * beta_i + s * ((2^q - 1)/2 - z):
#   alpha_i = s * 2^(i-1) (plane i = bit i of c, 0-based) and
#   offset  = s * ((2^q - 1)/2 - z).
# ---------------------------------------------------------------------------
def uniform_to_bcq(codes, scale, zero, q: int, g: int):
    """Rewrite a uniform q-bit weight as BCQ.

    codes uint8 [m][n] in [0, 2^q); scale fp16 [n/g][m]; zero uint8 [n/g][m]
    in [0, 2^q).  Returns (signs int8 [q][m][n], alpha fp16 [q][n/g][m],
    offset fp32 [n/g][m]).  alpha_i = RNE_fp16(s * 2^(i-1)) (exact unless s*2^-1
    is an fp16 subnormal with its last bit set); offset = s * ((2^q-1)/2 - z),
    exact in fp32 (an 11-bit significand times a half-integer below 2^q).
    """
    c = np.asarray(codes, dtype=np.int64)
    z = np.asarray(zero, dtype=np.int64)
    s64 = np.asarray(scale, dtype=np.float16).astype(np.float64)
    m, n = c.shape
    top = 1 << q
    if c.min(initial=0) < 0 or c.max(initial=0) >= top:
        raise ValueError("codes must lie in [0, 2^q)")
    if z.min(initial=0) < 0 or z.max(initial=0) >= top:
        raise ValueError("zero-points must lie in [0, 2^q)")
    signs = np.empty((q, m, n), dtype=np.int8)
    alpha = np.empty((q,) + s64.shape, dtype=np.float16)
    for i in range(q):
        signs[i] = (((c >> i) & 1) * 2 - 1).astype(np.int8)
        alpha[i] = (s64 * (2.0 ** (i - 1))).astype(np.float16)
    offset = (s64 * ((top - 1) / 2.0 - z)).astype(np.float32)
    return signs, alpha, offset


def uniform_dequant(codes, scale, zero, g: int) -> np.ndarray:
    """The plain uniform dequantisation w[j,k] = s[k//g, j] * (c[j,k] - z[k//g, j]) in FP64."""
    c = np.asarray(codes, dtype=np.float64)
    s = np.repeat(np.asarray(scale, dtype=np.float16).astype(np.float64), g, axis=0).T
    z = np.repeat(np.asarray(zero, dtype=np.float64), g, axis=0).T
    return s * (c - z)


# ---------------------------------------------------------------------------
# BCQ fitting: FP16 weights -> q sign planes and group scales (the step before
# the lookup path).  The pages only cite the method (LUT-GEMM card, reference
# 48: "Alternating multi-bit quantization"; Summary: weights are stored in
# BCQ).  Reading used here, per (row j, group G of g inputs), in FP64:
#   1. greedy: r = w; for i = 0..q-1: beta_i = sign(r) (sign(0) = +1),
#      alpha_i = mean(beta_i * r) = mean|r|, r -= alpha_i * beta_i;
#   2. `iters` rounds of
#      a. alpha-step: least squares alpha = argmin |w - B alpha|^2 with the
#         signs B (g x q) fixed, by Cholesky of B^T B; a pivot <= 1e-6 * g
#         (planes linearly dependent on the group) keeps the previous alpha;
#      b. beta-step: each input independently takes the sign combination
#         whose value sum_i alpha_i s_i is nearest to w (ties: the largest
#         code c, where bit i of c set means s_i = +1, so w = 0 at q = 1
#         keeps the greedy sign +1);
#   3. alpha is rounded to FP16 and a last beta-step uses the rounded alpha, so
#      the stored signs are the best ones for the stored scales.
# Each alpha-step and beta-step can only lower |w - B alpha|^2.
# ---------------------------------------------------------------------------
PIVOT_REL = 1e-6


def _code_signs(q: int) -> np.ndarray:
    """[2^q][q] sign matrix: row c has s_i = +1 iff bit i of c is set."""
    c = np.arange(1 << q)[:, None]
    return np.where((c >> np.arange(q)[None, :]) & 1, 1.0, -1.0)


def nearest_codes(w_groups, alpha):
    """beta-step.  w_groups [..., g], alpha [q, ...] -> signs [q, ..., g] (+-1.0)."""
    a = np.asarray(alpha, dtype=np.float64)
    q = a.shape[0]
    S = _code_signs(q)                                   # [C][q]
    vals = np.einsum("cq,q...->...c", S, a)              # [..., C]
    d = np.abs(np.asarray(w_groups, dtype=np.float64)[..., :, None] - vals[..., None, :])
    C = S.shape[0]
    best = C - 1 - np.argmin(d[..., ::-1], axis=-1)      # ties: the largest code
    return np.moveaxis(S[best], -1, 0)                   # [q, ..., g]


def _ls_alpha(w_groups, B, a_old, g: int):
    """alpha-step: Cholesky solve of (B^T B) alpha = B^T w per group."""
    q = B.shape[0]
    M = np.einsum("i...k,j...k->...ij", B, B)
    v = np.einsum("i...k,...k->...i", B, w_groups)
    L = np.zeros(M.shape)
    ok = np.ones(M.shape[:-2], dtype=bool)
    for i in range(q):
        for j in range(i + 1):
            acc = M[..., i, j] - np.einsum("...k,...k->...", L[..., i, :j], L[..., j, :j])
            if i == j:
                ok &= acc > PIVOT_REL * g
                L[..., i, i] = np.sqrt(np.maximum(acc, PIVOT_REL * g))
            else:
                L[..., i, j] = acc / L[..., j, j]
    y = np.zeros(v.shape)
    for i in range(q):                                   # L y = v
        y[..., i] = (v[..., i] - np.einsum("...k,...k->...", L[..., i, :i], y[..., :i])) / L[..., i, i]
    a = np.zeros(v.shape)
    for i in reversed(range(q)):                         # L^T a = y
        a[..., i] = (y[..., i] - np.einsum("...k,...k->...", L[..., i + 1:, i], a[..., i + 1:])) / L[..., i, i]
    a = np.moveaxis(a, -1, 0)
    return np.where(ok[None], a, a_old)


def _fit_groups(w, q: int, g: int, iters: int, trace=None):
    W = np.asarray(w, dtype=np.float64)
    m, n = W.shape
    if n % g != 0:
        raise ValueError("n % g != 0")
    Wg = W.reshape(m, n // g, g)
    r = Wg.copy()
    B = np.empty((q,) + Wg.shape)
    a = np.empty((q,) + Wg.shape[:-1])
    for i in range(q):
        B[i] = np.where(r >= 0, 1.0, -1.0)
        a[i] = (B[i] * r).sum(-1) / g
        r -= a[i][..., None] * B[i]
    if trace is not None:
        trace.append(((Wg - np.einsum("i...,i...k->...k", a, B)) ** 2).sum(-1))
    for _ in range(iters):
        a = _ls_alpha(Wg, B, a, g)
        if trace is not None:
            trace.append(((Wg - np.einsum("i...,i...k->...k", a, B)) ** 2).sum(-1))
        B = nearest_codes(Wg, a)
        if trace is not None:
            trace.append(((Wg - np.einsum("i...,i...k->...k", a, B)) ** 2).sum(-1))
    return Wg, a, B


def fit_bcq(w, q: int, g: int, iters: int):
    """FP16 W [m][n] -> (signs int8 [q][m][n], alpha fp16 [q][n/g][m],
    squared error per group fp64 [n/g][m] of the stored result)."""
    Wg, a, _ = _fit_groups(w, q, g, iters)
    a16 = a.astype(np.float16)
    B = nearest_codes(Wg, a16.astype(np.float64))
    err = ((Wg - np.einsum("i...,i...k->...k", a16.astype(np.float64), B)) ** 2).sum(-1)
    m, ng, _ = Wg.shape
    signs = B.reshape(q, m, ng * g).astype(np.int8)
    return signs, np.ascontiguousarray(np.transpose(a16, (0, 2, 1))), np.ascontiguousarray(err.T)


def fit_bcq_trace(w, q: int, g: int, iters: int):
    """Squared error per group after the greedy pass and after every alpha- and
    beta-step (unrounded alpha), as a list of [m][n/g] arrays."""
    trace = []
    _fit_groups(w, q, g, iters, trace)
    return trace


# ---------------------------------------------------------------------------
# Variable-grid fitting: the BCQ planes plus one constant per (row, group),
#   w ~ off + sum_i alpha_i * beta_i,
# a grid of 2^q points built from bit-planes and scalar coefficients (BPDQ
# card: "variable quantization grids from bit-planes and scalar
# coefficients"; the pages give no more than that line).  It is the format
# lutgemm_run consumes with an offset.  Reading used here, per (row, group):
#   1. greedy: off = mean(w), r = w - off, then the BCQ greedy planes on r;
#   2. `iters` rounds of
#      a. least squares for (alpha_0 .. alpha_{q-1}, off) with the signs
#         fixed: the columns are the q sign planes and a column of ones, the
#         unknowns in that order; Cholesky of the (q+1) x (q+1) normal matrix,
#         the same pivot rule (a dependent column keeps the previous values);
#      b. each input takes the grid point off + sum_i alpha_i s_i nearest to w
#         (ties: the largest code);
#   3. alpha rounded to fp16, off to fp32 (the offset type lutgemm_run reads),
#      then a last nearest-point step with the stored values.
# At q = 1 this is Lloyd's algorithm for two levels in one dimension.
# ---------------------------------------------------------------------------
def nearest_grid_codes(w_groups, alpha, off):
    """Nearest grid point off + sum_i alpha_i s_i.  w_groups [..., g],
    alpha [q, ...], off [...] -> signs [q, ..., g] (+-1.0); ties: the largest code."""
    a = np.asarray(alpha, dtype=np.float64)
    S = _code_signs(a.shape[0])                               # [C][q]
    vals = np.asarray(off, dtype=np.float64)[..., None] + np.einsum("cq,q...->...c", S, a)   # [..., C]
    d = np.abs(np.asarray(w_groups, dtype=np.float64)[..., :, None] - vals[..., None, :])
    C = S.shape[0]
    best = C - 1 - np.argmin(d[..., ::-1], axis=-1)
    return np.moveaxis(S[best], -1, 0)


def _ls_grid(w_groups, B, a_old, off_old, g: int):
    """Least squares for (alpha, off): the sign planes and a ones column."""
    ones = np.ones((1,) + B.shape[1:])
    coef = _ls_alpha(w_groups, np.concatenate([B, ones], axis=0),
                     np.concatenate([a_old, np.asarray(off_old)[None]], axis=0), g)
    return coef[:-1], coef[-1]


def _grid_value(a, off, B):
    return off[..., None] + np.einsum("i...,i...k->...k", a, B)


def _fit_groups_grid(w, q: int, g: int, iters: int, trace=None):
    W = np.asarray(w, dtype=np.float64)
    m, n = W.shape
    if n % g != 0:
        raise ValueError("n % g != 0")
    Wg = W.reshape(m, n // g, g)
    off = Wg.mean(-1)
    r = Wg - off[..., None]
    B = np.empty((q,) + Wg.shape)
    a = np.empty((q,) + Wg.shape[:-1])
    for i in range(q):
        B[i] = np.where(r >= 0, 1.0, -1.0)
        a[i] = (B[i] * r).sum(-1) / g
        r -= a[i][..., None] * B[i]
    if trace is not None:
        trace.append(((Wg - _grid_value(a, off, B)) ** 2).sum(-1))
    for _ in range(iters):
        a, off = _ls_grid(Wg, B, a, off, g)
        if trace is not None:
            trace.append(((Wg - _grid_value(a, off, B)) ** 2).sum(-1))
        B = nearest_grid_codes(Wg, a, off)
        if trace is not None:
            trace.append(((Wg - _grid_value(a, off, B)) ** 2).sum(-1))
    return Wg, a, off, B


def fit_bcq_grid(w, q: int, g: int, iters: int):
    """FP16 W [m][n] -> (signs int8 [q][m][n], alpha fp16 [q][n/g][m],
    offset fp32 [n/g][m], squared error per group fp64 [n/g][m] of the stored result)."""
    Wg, a, off, _ = _fit_groups_grid(w, q, g, iters)
    a16 = a.astype(np.float16)
    off32 = off.astype(np.float32)
    B = nearest_grid_codes(Wg, a16.astype(np.float64), off32.astype(np.float64))
    err = ((Wg - _grid_value(a16.astype(np.float64), off32.astype(np.float64), B)) ** 2).sum(-1)
    m, ng, _ = Wg.shape
    signs = B.reshape(q, m, ng * g).astype(np.int8)
    return (signs, np.ascontiguousarray(np.transpose(a16, (0, 2, 1))), np.ascontiguousarray(off32.T),
            np.ascontiguousarray(err.T))


def fit_bcq_grid_trace(w, q: int, g: int, iters: int):
    """Squared error per group after the greedy pass and after every step (unrounded values)."""
    trace = []
    _fit_groups_grid(w, q, g, iters, trace)
    return trace


# ---------------------------------------------------------------------------
# Mixed storage: 2-, 4- and 16-bit weights in one matrix (OpenAlex record
# "Fast and Efficient 2-bit LLM Inference on GPU: 2/4/16-bit in a Weight
# Matrix with Asynchronous Dequantization", abstract: weights are quantised
# by groups, some groups hold a large range, and sparse outliers are kept at
# higher precision).  The record gives the idea only (its abstract stops at
# the problem statement).  Reading used here, in BCQ form:
#   * a precision block (s, R) is rows 32R .. 32R+31 by inputs 1024s ..
#     1024s+1023, the unit the lookup kernel streams; it carries q_b planes,
#     1 <= q_b <= q_max (2 planes for most blocks, 4 for wide-range ones);
#   * W[j,k] = sum_{i < q_b(j // 32, k // 1024)} alpha[i, k // g, j] * beta[i, j, k]
#              + S[j, k],
#     where S is a sparse fp16 matrix, the 16-bit outliers, ADDED to the
#     BCQ value (a sign plane has no zero, so the BCQ part cannot leave a
#     position out; a fitter stores the outlier's residual);
#   * packed planes: blocks in (s, R) order, block (s, R) holds q_b * 4096
#     bytes from byte 4096 * off[s * m_t + R], off the exclusive prefix sum
#     of q_b in that order; inside a block the planes are stored in pairs:
#     pair h holds planes 2h and 2h+1 (only 2h when q_b = 2h + 1), e_h of
#     them, from byte 8192 * h of the block, and its chunk (U, i') (plane
#     2h + i') sits at (U * e_h + i') * 512 from there, with the byte map of
#     the uniform layout (so a block of at most two planes is laid out as
#     pack_bcq lays it out; pairs let the kernel move two planes per copy
#     whatever the block's count);
#   * outliers for the kernel: slice-major CSR, the entries of (slice s,
#     row r) at [optr[s * m + r], optr[s * m + r + 1]), sorted by input, each
#     a uint32 (k - 1024 s) | (fp16 bits << 16).
# block_planes is uint8 [n_s][m_t]; outliers are given as row CSR
# (row_ptr [m + 1], col [nnz] increasing within a row, val fp16 [nnz]).
# ---------------------------------------------------------------------------
def _check_blocks(block_planes, m: int, n: int):
    bp = np.asarray(block_planes, dtype=np.int64)
    ns, mt = math.ceil(n / SLICE), math.ceil(m / TILE_ROWS)
    if bp.shape != (ns, mt):
        raise ValueError(f"block_planes must be [{ns}][{mt}]")
    if bp.min(initial=1) < 1:
        raise ValueError("every block needs at least one plane")
    return bp


def mixed_block_offsets(block_planes) -> np.ndarray:
    """Exclusive prefix sum of the plane counts in (s, R) order, in 4096-byte
    blocks: uint32 [n_s * m_t + 1]; the last entry is the total."""
    bp = np.asarray(block_planes, dtype=np.int64).reshape(-1)
    return np.concatenate([[0], np.cumsum(bp)]).astype(np.uint32)


def mixed_packed_nbytes(block_planes) -> int:
    return int(np.asarray(block_planes, dtype=np.int64).sum()) * BLOCK_BYTES


def _plane_pairs(qb: int):
    """(first plane, planes) of each stored pair of a block with qb planes."""
    return [(2 * h, min(2, qb - 2 * h)) for h in range((qb + 1) // 2)]


def pack_mixed(signs, block_planes) -> np.ndarray:
    """int8 signs [q_max][m][n] -> the mixed packed buffer.  Block (s, R)
    stores planes 0 .. q_b - 1 of its rows and inputs, pair by pair, each
    pair packed as a one-tile, one-slice matrix by ``pack_bcq``; planes from
    q_b on are not stored."""
    sg = np.asarray(signs)
    q_max, m, n = sg.shape
    bp = _check_blocks(block_planes, m, n)
    if bp.max(initial=1) > q_max:
        raise ValueError("a block has more planes than signs were given")
    ns, mt = bp.shape
    parts = []
    for s_ in range(ns):
        for R in range(mt):
            qb = int(bp[s_, R])
            for i0, e in _plane_pairs(qb):
                blk = sg[i0: i0 + e, TILE_ROWS * R: TILE_ROWS * (R + 1), SLICE * s_: SLICE * (s_ + 1)]
                parts.append(pack_bcq(blk))
    return np.concatenate(parts)


def unpack_mixed(packed, block_planes, q_max: int, m: int, n: int) -> np.ndarray:
    """Inverse of ``pack_mixed``: signs int8 [q_max][m][n], with 0 where a
    block stores no plane."""
    pk = np.asarray(packed, dtype=np.uint8).reshape(-1)
    bp = _check_blocks(block_planes, m, n)
    assert pk.size == mixed_packed_nbytes(bp)
    off = mixed_block_offsets(bp)
    ns, mt = bp.shape
    out = np.zeros((q_max, m, n), dtype=np.int8)
    for s_ in range(ns):
        for R in range(mt):
            u = s_ * mt + R
            qb = int(bp[s_, R])
            r0, k0 = TILE_ROWS * R, SLICE * s_
            mr, nk = min(m, r0 + TILE_ROWS) - r0, min(n, k0 + SLICE) - k0
            base = int(off[u]) * BLOCK_BYTES
            for i0, e in _plane_pairs(qb):
                blk = pk[base + i0 * BLOCK_BYTES: base + (i0 + e) * BLOCK_BYTES]
                out[i0: i0 + e, r0: r0 + mr, k0: k0 + nk] = unpack_bcq_vec(blk, e, mr, nk)
    return out


def outlier_dense(row_ptr, col, val, m: int, n: int) -> np.ndarray:
    """The sparse outlier matrix S as a dense FP64 [m][n] array."""
    rp = np.asarray(row_ptr, dtype=np.int64)
    c = np.asarray(col, dtype=np.int64)
    v = np.asarray(val, dtype=np.float16).astype(np.float64)
    S_ = np.zeros((m, n), dtype=np.float64)
    for r in range(m):
        ks = c[rp[r]: rp[r + 1]]
        if np.any(np.diff(ks) <= 0) or (ks.size and (ks.min() < 0 or ks.max() >= n)):
            raise ValueError("outlier columns must increase within a row and lie in [0, n)")
        S_[r, ks] = v[rp[r]: rp[r + 1]]
    return S_


def mixed_weights(signs, alpha, block_planes, g: int, outliers=None) -> np.ndarray:
    """The plain FP64 W of the mixed format (definition above).

    signs [q_max][m][n] (planes a block does not store are ignored);
    alpha [q_max][n/g][m]; outliers None or (row_ptr, col, val)."""
    sg = np.asarray(signs)
    q_max, m, n = sg.shape
    bp = _check_blocks(block_planes, m, n)
    a = np.asarray(alpha, dtype=np.float64)
    assert a.shape == (q_max, n // g, m)
    qb = np.repeat(np.repeat(bp.T, TILE_ROWS, axis=0)[:m], SLICE, axis=1)[:, :n]   # [m][n]
    W = np.zeros((m, n), dtype=np.float64)
    for i in range(q_max):
        a_rows = np.repeat(a[i], g, axis=0).T
        W += np.where(i < qb, a_rows * sg[i].astype(np.float64), 0.0)
    if outliers is not None:
        W += outlier_dense(*outliers, m, n)
    return W


def mixed_matmul(x, signs, alpha, block_planes, g: int, outliers=None) -> np.ndarray:
    """y[b, j] = sum_k W[j, k] x[b, k] with W from ``mixed_weights``; FP64 [batch][m]."""
    return np.asarray(x, dtype=np.float64) @ mixed_weights(signs, alpha, block_planes, g, outliers).T


def pack_outliers(row_ptr, col, val, m: int, n: int):
    """Row CSR outliers -> (optr uint32 [n_s * m + 1], oent uint32 [nnz]): the
    slice-major layout above."""
    rp = np.asarray(row_ptr, dtype=np.int64)
    c = np.asarray(col, dtype=np.int64)
    bits = np.asarray(val, dtype=np.float16).view(np.uint16).astype(np.uint32)
    ns = math.ceil(n / SLICE)
    outlier_dense(rp, c, np.asarray(val, dtype=np.float16), m, n)     # validates the CSR
    optr = np.zeros(ns * m + 1, dtype=np.uint32)
    ent = []
    for s_ in range(ns):
        for r in range(m):
            e = np.arange(rp[r], rp[r + 1])
            e = e[(c[e] >= SLICE * s_) & (c[e] < SLICE * (s_ + 1))]
            ent.extend(((c[e] - SLICE * s_) | (bits[e] << 16)).tolist())
            optr[s_ * m + r + 1] = len(ent)
    return optr, np.asarray(ent, dtype=np.uint32)


def unpack_outliers(optr, oent, m: int, n: int) -> np.ndarray:
    """Inverse of ``pack_outliers``, as a dense FP64 [m][n] array."""
    optr = np.asarray(optr, dtype=np.int64)
    oent = np.asarray(oent, dtype=np.uint32)
    ns = math.ceil(n / SLICE)
    S_ = np.zeros((m, n), dtype=np.float64)
    for s_ in range(ns):
        for r in range(m):
            for e in range(optr[s_ * m + r], optr[s_ * m + r + 1]):
                k = SLICE * s_ + int(oent[e] & 0xFFFF)
                S_[r, k] = float(np.uint16(oent[e] >> 16).view(np.float16))
    return S_


def mixed_matmul_tiles(x, packed, block_planes, alpha, g: int, m: int, n: int, tiles, outliers=None):
    """``mixed_matmul`` restricted to the rows of the given row tiles, read
    straight from a mixed packed buffer: each block of those tiles is
    unpacked, the rows' scales and outliers are taken, and the product is the
    plain definition on that sub-matrix.  Returns (y [batch][rows], rows)."""
    pk = np.asarray(packed, dtype=np.uint8).reshape(-1)
    bp = _check_blocks(block_planes, m, n)
    off = mixed_block_offsets(bp)
    a = np.asarray(alpha)
    q_max = a.shape[0]
    ns, mt = bp.shape
    tiles = np.asarray(tiles, dtype=np.int64)
    rows = (TILE_ROWS * tiles[:, None] + np.arange(TILE_ROWS)[None, :]).reshape(-1)
    rows = rows[rows < m]
    signs = np.zeros((q_max, rows.size, n), dtype=np.int8)
    r0 = 0
    for R in tiles:
        mr = min(m, TILE_ROWS * (int(R) + 1)) - TILE_ROWS * int(R)
        for s_ in range(ns):
            u = s_ * mt + int(R)
            qb = int(bp[s_, R])
            k0 = SLICE * s_
            nk = min(n, k0 + SLICE) - k0
            base = int(off[u]) * BLOCK_BYTES
            for i0, e in _plane_pairs(qb):
                blk = pk[base + i0 * BLOCK_BYTES: base + (i0 + e) * BLOCK_BYTES]
                signs[i0: i0 + e, r0: r0 + mr, k0: k0 + nk] = unpack_bcq_vec(blk, e, mr, nk)
        r0 += mr
    sub = None
    if outliers is not None:
        rp, col, val = (np.asarray(t) for t in outliers)
        sub_rp, sub_col, sub_val = [0], [], []
        for r in rows:
            sub_col.extend(col[rp[r]: rp[r + 1]].tolist())
            sub_val.extend(val[rp[r]: rp[r + 1]].tolist())
            sub_rp.append(len(sub_col))
        sub = (np.asarray(sub_rp), np.asarray(sub_col, dtype=np.int64), np.asarray(sub_val, dtype=np.float16))
    # The sub-matrix's row tiles are the chosen tiles in order, so its block
    # plane counts are those columns of block_planes.
    y = mixed_matmul(x, signs, a[:, :, rows], bp[:, tiles], g, sub)
    return y, rows


# ---------------------------------------------------------------------------
# Unit-major scales of mixed storage (this library's own layout, defined in
# include/lutgemm.h): the scales of the planes each block stores, in the
# order the kernel's lanes read them.  For g % 128 == 0 (H = 1) and g == 64
# (H = 2).  Block u = s * m_t + R with table entry off[u] starts at element
# off[u] * 256 * H; its pair h (planes 2h and 2h+1, or 2h alone; e_h planes)
# at + h * 512 * H; lane l's pass at + l * 8 * e_h * H; element
# (U * e_h + e) * H + hh of it holds alpha[2h + e][G][32R + l] with
# G = (1024 s + 128 P + 64 hh) // g, P = U xor 4 * (l // 16); 0 for rows >= m
# or inputs >= n.  With every block at q <= 2 planes this is pack_scales's
# buffer for those q planes.
# ---------------------------------------------------------------------------
def mixed_scales_nbytes(block_planes, g: int) -> int:
    H = 2 if g == PIECE // 2 else 1
    return int(np.asarray(block_planes, dtype=np.int64).sum()) * 512 * H


def pack_mixed_scales(alpha, block_planes, g: int) -> np.ndarray:
    """fp16 alpha [q_max][n/g][m] -> fp16 unit-major mixed scale buffer (1-D)."""
    a = np.asarray(alpha, dtype=np.float16)
    q_max, ng, m = a.shape
    n = ng * g
    if not (g % PIECE == 0 or g == PIECE // 2):
        raise ValueError("unit-major scales need g % 128 == 0 or g == 64")
    H = 2 if g == PIECE // 2 else 1
    bp = _check_blocks(block_planes, m, n)
    off = mixed_block_offsets(bp)
    ns, mt = bp.shape
    out = np.zeros(int(off[-1]) * 256 * H, dtype=np.float16)
    for s_ in range(ns):
        for R in range(mt):
            u = s_ * mt + R
            base = int(off[u]) * 256 * H
            for i0, e_h in _plane_pairs(int(bp[s_, R])):
                h = i0 // 2
                for l in range(TILE_ROWS):
                    row = TILE_ROWS * R + l
                    if row >= m:
                        continue
                    for U in range(8):
                        P = U ^ (4 * (l // 16))
                        for hh in range(H):
                            k0 = SLICE * s_ + PIECE * P + (PIECE // 2) * hh
                            if k0 >= n:
                                continue
                            for e in range(e_h):
                                idx = base + h * 512 * H + l * 8 * e_h * H + (U * e_h + e) * H + hh
                                out[idx] = a[i0 + e, k0 // g, row]
    return out


def unpack_mixed_scales(scales, block_planes, q_max: int, m: int, n: int, g: int) -> np.ndarray:
    """Inverse of ``pack_mixed_scales``: alpha [q_max][n/g][m] with the scales
    the blocks store (a group wider than a piece appears once per piece; the
    copies must agree) and 0 for planes no block of the group stores."""
    H = 2 if g == PIECE // 2 else 1
    bp = _check_blocks(block_planes, m, n)
    off = mixed_block_offsets(bp)
    buf = np.asarray(scales, dtype=np.float16)
    ns, mt = bp.shape
    out = np.zeros((q_max, n // g, m), dtype=np.float64)
    seen = np.zeros(out.shape, dtype=bool)
    for s_ in range(ns):
        for R in range(mt):
            u = s_ * mt + R
            base = int(off[u]) * 256 * H
            for i0, e_h in _plane_pairs(int(bp[s_, R])):
                h = i0 // 2
                for l in range(TILE_ROWS):
                    row = TILE_ROWS * R + l
                    if row >= m:
                        continue
                    for U in range(8):
                        P = U ^ (4 * (l // 16))
                        for hh in range(H):
                            k0 = SLICE * s_ + PIECE * P + (PIECE // 2) * hh
                            if k0 >= n:
                                continue
                            for e in range(e_h):
                                v = float(buf[base + h * 512 * H + l * 8 * e_h * H + (U * e_h + e) * H + hh])
                                G = k0 // g
                                if seen[i0 + e, G, row] and out[i0 + e, G, row] != v:
                                    raise ValueError("copies of one group scale disagree")
                                out[i0 + e, G, row] = v
                                seen[i0 + e, G, row] = True
    return out.astype(np.float16)
