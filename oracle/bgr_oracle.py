"""CPU oracle of bounded-init grid refinement (BGR) for the weights.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only the test-suite, the smoke check and the CPU-baseline
leg of the benchmark use it.  It shares no code with the CUDA library.

What the pages fix (DVD-Quant, "Resumen técnico" §2.A, "Refinamiento de
Rejilla con Inicialización Acotada"; the lay summary's point 1 says the same):
DiT weights are close to Gaussian, so a MinMax grid wastes levels on the rare
extreme values.  BGR first searches for bounds that progressively exclude
outliers, then refines the quantization step Δ and the zero point z
iteratively, each time by the closed-form least-squares fit that minimises
the quantization error.  It runs offline, on the weights only.

Readings taken where the pages are silent (the pages give no formula, count
or schedule):

* Grid: asymmetric, b bits, levels q in [0, 2^b - 1], dequantised value
  Δ (q - z) with an integer zero point z in [0, 2^b - 1] (so that 0 is a
  level).  It applies per output channel to the rotated weight row u (the
  binary32 block Walsh-Hadamard transform of the bf16 row, as in the
  symmetric path; the 2^-7 of the two normalisations is folded into the
  stored scale).
* Codes for a grid: inv = fl(1 / Δ) (one binary64 division), then
  q = clamp(rint_half_even(fl(u · inv)) + z, 0, 2^b - 1), binary64.
* Error of a grid: E = sum_k (u_k - fl(Δ (q_k - z)))^2, every step one binary64
  operation (no fused multiply-add), summed in index order.
* Bound search ("excluding outliers progressively"): for j = 0..J-1 the
  candidate bounds are r_j·[min u, max u] with r_j = 1 - j/(2J) (from the full
  range down to a little over half of it); the candidate's grid is
  Δ = fl((hi - lo) / (2^b - 1)), z = clamp(rint(fl(-lo / Δ)), 0, 2^b - 1).
  The candidate with the smallest E wins (the first one on ties).  A row with
  max u == min u gets the one-level grid Δ = |u_0| (or 1 if u_0 = 0), z chosen
  so that u_0 is a level when possible.
* Refinement, T iterations: given the codes q of the current grid, the
  closed-form least-squares fit of u ≈ Δ q + c over (Δ, c) (sums in index
  order, binary64), z = clamp(rint(-c / Δ), 0, 2^b - 1) (integer zero point),
  then Δ refit for that z: Δ = sum u (q - z) / sum (q - z)^2; the row is
  re-quantised with the new grid.  The grid with the smallest E over the
  initial one and all iterations is kept (so the error never grows).  A
  degenerate fit (zero denominator or Δ <= 0) ends the iterations.
* Storage: signed codes s = q - 2^(b-1) (int4 nibbles or int8 bytes, the same
  packing as the symmetric path), the stored scale fl32(Δ)·2^-7 and an integer
  offset o = 2^(b-1) - z, so Δ (q - z) = Δ (s + o).
* Layer: acc = sum_k q_a[m,k] s[n,k] + o[n] · sum_k q_a[m,k] (exact integers),
  then the same epilogue as the symmetric layer.
"""

from __future__ import annotations

import numpy as np

from .qs_oracle import (bf16_bits_to_f32, epilogue, fwht128_blocks, int_gemm, pack,
                        quant_act)

BGR_DEFAULT_CANDIDATES = 64
BGR_DEFAULT_ITERATIONS = 8


def seq_sum(v: np.ndarray) -> float:
    """Sum in index order, binary64 (each partial sum rounded once)."""
    v = np.asarray(v, dtype=np.float64)
    return float(np.cumsum(v)[-1]) if v.size else 0.0


def grid_codes(u: np.ndarray, delta: float, z: int, bits: int) -> np.ndarray:
    """q = clamp(rint(fl(u * fl(1/Δ))) + z, 0, 2^b - 1) in binary64."""
    inv = np.float64(1.0) / np.float64(delta)
    r = np.rint(np.asarray(u, dtype=np.float64) * inv)
    return np.clip(r + z, 0, (1 << bits) - 1).astype(np.int64)


def grid_error(u: np.ndarray, delta: float, z: int, q: np.ndarray) -> float:
    """E = sum_k (u_k - fl(Δ (q_k - z)))^2 in index order, binary64."""
    dq = np.float64(delta) * (q - z).astype(np.float64)
    e = np.asarray(u, dtype=np.float64) - dq
    return seq_sum(e * e)


def grid_from_bounds(lo: float, hi: float, bits: int) -> tuple[float, int]:
    levels = (1 << bits) - 1
    delta = (np.float64(hi) - np.float64(lo)) / np.float64(levels)
    z = int(np.clip(np.rint(-np.float64(lo) / delta), 0, levels))
    return float(delta), z


def _flat_grid(u0: float, bits: int) -> tuple[float, int]:
    """One-level row: Δ = |u0| (1 if u0 = 0); u0 = Δ (q - z) with q = z ± 1 or z."""
    levels = (1 << bits) - 1
    if u0 == 0.0:
        return 1.0, 0
    return abs(float(u0)), (0 if u0 > 0 else levels)


def bound_search(u: np.ndarray, bits: int, candidates: int) -> tuple[float, int, float]:
    """The bounded initialisation: the best of the shrunk MinMax grids."""
    lo, hi = float(np.min(u)), float(np.max(u))
    if hi == lo:
        d, z = _flat_grid(lo, bits)
        return d, z, grid_error(u, d, z, grid_codes(u, d, z, bits))
    best = None
    for j in range(candidates):
        r = 1.0 - j / (2.0 * candidates)
        d, z = grid_from_bounds(r * lo, r * hi, bits)
        e = grid_error(u, d, z, grid_codes(u, d, z, bits))
        if best is None or e < best[2]:
            best = (d, z, e)
    return best


def least_squares_grid(u: np.ndarray, q: np.ndarray, bits: int) -> tuple[float, int] | None:
    """The closed-form fit u ≈ Δ q + c, then the integer zero point and Δ refit."""
    levels = (1 << bits) - 1
    u = np.asarray(u, dtype=np.float64)
    qf = q.astype(np.float64)
    n = float(u.size)
    sq, sqq = float(np.sum(q)), float(np.sum(q * q))        # exact integers
    su, squ = seq_sum(u), seq_sum(qf * u)                   # products exact in binary64
    den = n * sqq - sq * sq
    if den == 0.0:
        return None
    delta = (n * squ - sq * su) / den
    if not delta > 0.0:
        return None
    c = (su - delta * sq) / n
    z = int(np.clip(np.rint(-c / delta), 0, levels))
    t = qf - float(z)
    tt = float(np.sum((q - z) * (q - z)))                   # exact integer
    if tt == 0.0:
        return None
    delta = seq_sum(u * t) / tt
    if not delta > 0.0:
        return None
    return float(delta), z


def bgr_row(u: np.ndarray, bits: int, candidates: int = BGR_DEFAULT_CANDIDATES,
            iterations: int = BGR_DEFAULT_ITERATIONS):
    """BGR of one row: returns (Δ, z, q, E) of the best grid found."""
    u = np.asarray(u, dtype=np.float64)
    d, z, e = bound_search(u, bits, candidates)
    best = (d, z, grid_codes(u, d, z, bits), e)
    cur_q = best[2]
    for _ in range(iterations):
        fit = least_squares_grid(u, cur_q, bits)
        if fit is None:
            break
        d, z = fit
        cur_q = grid_codes(u, d, z, bits)
        e = grid_error(u, d, z, cur_q)
        if e < best[3]:
            best = (d, z, cur_q, e)
    return best


def pack_weights_bgr(w_bits, bits: int, candidates: int = BGR_DEFAULT_CANDIDATES,
                     iterations: int = BGR_DEFAULT_ITERATIONS, rotate: bool = True):
    """Rotated weight rows on BGR grids: signed codes s = q - 2^(b-1) [N, K],
    stored scales fl32(Δ)·2^-7 (or fl32(Δ) without rotation) and offsets o."""
    w = bf16_bits_to_f32(np.asarray(w_bits))
    u = fwht128_blocks(w) if rotate else w
    N, K = u.shape
    half = 1 << (bits - 1)
    s = np.empty((N, K), np.int8)
    scale = np.empty(N, np.float32)
    offset = np.empty(N, np.int32)
    for n in range(N):
        d, z, q, _ = bgr_row(u[n].astype(np.float64), bits, candidates, iterations)
        s[n] = (q - half).astype(np.int8)
        scale[n] = np.float32(d) * (np.float32(2.0 ** -7) if rotate else np.float32(1.0))
        offset[n] = half - z
    return s, scale, offset


def code_rowsums(qa: np.ndarray) -> np.ndarray:
    """sum_k q_a[m, k] per token (exact)."""
    return np.asarray(qa, dtype=np.int64).sum(axis=1)


def asym_accumulators(qa: np.ndarray, s: np.ndarray, offset: np.ndarray,
                      gemm=int_gemm) -> np.ndarray:
    """acc[m, n] = sum_k q_a[m,k] s[n,k] + o[n] sum_k q_a[m,k]  (= sum q_a (q - z)).

    `gemm`: the exact integer product (int_gemm, or int_gemm_f64 -- exact by
    the 2^53 bound it checks -- for full-size operands)."""
    acc = gemm(qa, s) + code_rowsums(qa)[:, None] * np.asarray(offset, np.int64)[None, :]
    if np.abs(acc).max(initial=0) >= 2 ** 31:
        raise OverflowError("accumulator exceeds int32")
    return acc


def qlinear_bgr(x_bits, w_bits, bias_bits, bits: int, alpha: float,
                candidates: int = BGR_DEFAULT_CANDIDATES,
                iterations: int = BGR_DEFAULT_ITERATIONS, rotate: bool = True):
    """The layer with symmetric per-token activations and BGR weights."""
    qa, sa = quant_act(x_bits, bits, alpha, rotate)
    s, sw, off = pack_weights_bgr(w_bits, bits, candidates, iterations, rotate)
    acc = asym_accumulators(qa, s, off)
    out = epilogue(acc, sa, sw, bias_bits)
    return {"qa": qa, "sa": sa, "rowsum": code_rowsums(qa), "s": s, "sw": sw, "offset": off,
            "xp": pack(qa, bits), "wp": pack(s, bits), "acc": acc, "out": out}
