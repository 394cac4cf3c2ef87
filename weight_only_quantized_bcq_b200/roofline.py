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
