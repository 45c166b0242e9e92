"""Row-parallel evaluation of oracle functions for the full-size GPU tests.

Test infrastructure: the oracle's per-row work (the BGR grid search, the SD4
quantiser) takes minutes on one core at the full weight and activation sizes,
so it is split into row blocks evaluated by a pool of SPAWNED processes (the
test process holds a CUDA context; a forked child of it could hang).  Each
block is computed by the unchanged oracle function and the blocks are
concatenated in row order, so the result is the oracle's.
"""

from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np


def _bgr_block(args):
    wb, bits, candidates, iterations = args
    from oracle import bgr_oracle as B
    return B.pack_weights_bgr(wb, bits, candidates, iterations)


def _sd4_block(xb):
    from oracle import sd4_oracle as S
    return S.quantize_rows(xb)


def _sd4_decomp_block(xb):
    from oracle import sd4_oracle as S
    return S.decompose_rows(xb, range(len(xb)))


def _map(fn, items):
    procs = min(len(items), os.cpu_count() or 1)
    saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS")}
    for k in saved:
        os.environ[k] = "1"
    try:
        with mp.get_context("spawn").Pool(procs) as pool:
            return pool.map(fn, items, chunksize=1)
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


def _blocks(a: np.ndarray, n: int) -> list[np.ndarray]:
    return [np.ascontiguousarray(b) for b in np.array_split(a, n) if len(b)]


def bgr_pack_weights(w_bits: np.ndarray, bits: int, candidates: int, iterations: int):
    """oracle.bgr_oracle.pack_weights_bgr over row blocks: (codes, scales, offsets)."""
    parts = _map(_bgr_block, [(b, bits, candidates, iterations)
                              for b in _blocks(w_bits, 4 * (os.cpu_count() or 1))])
    return (np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts]),
            np.concatenate([p[2] for p in parts]))


def sd4_quantize_rows(x_bits: np.ndarray):
    """oracle.sd4_oracle.quantize_rows over row blocks: (codes, exponents, dialects)."""
    parts = _map(_sd4_block, _blocks(x_bits, 4 * (os.cpu_count() or 1)))
    return tuple(np.concatenate([p[i] for p in parts]) for i in range(3))


def sd4_decompose_rows(x_bits: np.ndarray) -> dict:
    """oracle.sd4_oracle.decompose_rows of every row of `x_bits`, over row
    blocks: the dict of per-row arrays, rows in order."""
    parts = _map(_sd4_decomp_block, _blocks(x_bits, 4 * (os.cpu_count() or 1)))
    return {k: np.concatenate([p[k] for p in parts]) for k in parts[0]}
