"""Oracle work for a pool of spawned CPU processes (test infrastructure).

Full-size parity checks compare every output of a large matmul with the FP64
oracle.  The rows are independent, so the oracle runs on chunks of row tiles
in parallel processes.  The processes are started with the "spawn" method
(a process forked from one that has used CUDA can hang), and this module
imports only numpy and the oracle.
"""
from __future__ import annotations

import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np


def _chunk(args):
    from oracle import bcq_oracle as O
    sub, q, m_sub, n, alpha_rows, x, g, offset_rows = args
    signs = O.unpack_bcq_vec(sub, q, m_sub, n)
    return O.bcq_matmul(x, signs, alpha_rows, g, offset_rows)


def oracle_all_rows(packed, q: int, m: int, n: int, alpha, x, g: int, offset=None, tiles_per_chunk: int = 64,
                    workers: int = None) -> np.ndarray:
    """y = W x for every row of a packed BCQ matrix, by the oracle, in parallel
    over chunks of row tiles.  packed: uint8 host buffer; alpha [q][n/g][m];
    x [batch][n]; offset [n/g][m] or None.  Returns [batch][m] fp64."""
    from oracle import bcq_oracle as O
    mt = -(-m // 32)
    jobs = []
    for R0 in range(0, mt, tiles_per_chunk):
        R1 = min(mt, R0 + tiles_per_chunk)
        sub, m_sub = O.packed_row_tiles(packed, q, m, n, R0, R1)
        rows = slice(32 * R0, 32 * R0 + m_sub)
        jobs.append((sub, q, m_sub, n, np.ascontiguousarray(alpha[:, :, rows]), x, g,
                     None if offset is None else np.ascontiguousarray(offset[:, rows])))
    workers = workers or max(1, min(len(jobs), os.cpu_count() or 1, 16))
    with ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn")) as ex:
        parts = list(ex.map(_chunk, jobs))
    return np.concatenate(parts, axis=1)
