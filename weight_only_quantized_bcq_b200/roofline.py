"""Byte accounting for the BCQ LUT-GEMM path (host arithmetic, no GPU).

Algorithmic bytes of one matmul are the bytes the method cannot avoid moving:
the q packed sign planes (q*m*n/8), the fp16 group scales (2*q*m*n/g), the
fp32 group offsets of converted uniform weights (4*m*n/g), the fp16 input x
(2*batch*n) and the fp32 output y (4*batch*m).  The weight part matches the
storage accounting of the LUT-GEMM card (Elamur, "Group size as a separate
hyper-parameter": scales count toward real storage), i.e. q + 16q/g bits per
weight.
"""
from __future__ import annotations


def bits_per_weight(q: int, g: int, with_offset: bool = False) -> float:
    """Storage bits per weight: q sign bits + 16q/g bits of fp16 scales (+32/g offset)."""
    return q + 16.0 * q / g + (32.0 / g if with_offset else 0.0)


def algorithmic_bytes(m: int, n: int, q: int, g: int, batch: int = 1,
                      with_offset: bool = False, y_bytes: int = 4) -> int:
    planes = q * m * n // 8
    alpha = 2 * q * m * (n // g)
    offset = 4 * m * (n // g) if with_offset else 0
    return planes + alpha + offset + 2 * batch * n + y_bytes * batch * m


def lookups(m: int, n: int, q: int, batch: int = 1) -> int:
    """Table reads of one matmul: one per (plane, row, 8-input run, batch column)."""
    return q * m * (n // 8) * batch


def mixed_algorithmic_bytes(block_planes, m: int, n: int, g: int, batch: int = 1, nnz: int = 0,
                            y_bytes: int = 4) -> int:
    """Bytes one product in mixed storage cannot avoid moving: the stored
    planes (4096 bytes per plane of every 32-row x 1024-input block), the fp16
    scales of the stored planes (one per plane, row and group of g inputs
    inside the block), the block table (4 bytes per block + 1), the outlier
    pointers (4 bytes per (slice, row) + 1) and entries (4 bytes each) when
    there are outliers, x and y.  block_planes: [n_s][m_t] plane counts."""
    ns, mt = -(-n // 1024), -(-m // 32)
    planes = 0
    scales = 0
    for s in range(ns):
        k0, k1 = 1024 * s, min(n, 1024 * (s + 1))
        groups = len(range(k0 // g, (k1 - 1) // g + 1))       # groups that meet this slice
        for R in range(mt):
            qb = int(block_planes[s][R])
            rows = min(m, 32 * (R + 1)) - 32 * R
            planes += 4096 * qb
            scales += 2 * qb * rows * groups
    table = 4 * (ns * mt + 1)
    outl = (4 * (ns * m + 1) + 4 * nnz) if nnz > 0 else 0
    return planes + scales + table + outl + 2 * batch * n + y_bytes * batch * m
