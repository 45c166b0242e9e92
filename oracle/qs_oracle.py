"""CPU oracle for the Hadamard-rotated W4A4 / W8A8 quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only the test-suite, the smoke check and the CPU-baseline
leg of the benchmark use it.  It shares no code, table or helper with the CUDA
library; the only thing both sides consume is the seeded synthetic input.

What is computed (DVD-Quant, "Resumen técnico" §2.B, "Cuantización Rotada con
Auto-Escalado (ARQ)"): a Hadamard rotation is applied to both the activations
and the weights, and the quantization scales are computed at run time from the
*rotated* activations, so no calibration set is needed.  The layer is W4A4
(§1 "Problema y Contexto", §4 "Resultados") or its 8-bit branch (§2.C,
"δ-GBS": the high-precision mode is 8 bits).

The pages leave the details open; the readings taken here are:

* Hadamard: Sylvester matrix of order 128 in natural order,
  H[i][j] = (-1)^popcount(i & j), applied to consecutive blocks of 128 along K
  (block size and the 1/sqrt(128) normalisation are the layer's stated
  parameters, not the pages').  The transform is the fast Walsh-Hadamard
  butterfly in binary32 with the stage order h = 1, 2, 4, ..., 64; at stage h
  every pair (i, i+h) with (i & h) == 0 becomes (a + b, a - b).  Fixing the
  stage order fixes every binary32 rounding, so the quantised codes are a
  deterministic function of the bf16 input.
* Normalisation folded into the scales: the codes are taken from the
  unnormalised u = x·H; the factor (1/sqrt(128))^2 = 2^-7 of the two rotations
  is exact in binary32 and is carried by the weight scale.
* Scale granularity: one scale per token (row of x) over the whole K row for
  activations, one per output channel (row of W) for weights.  A per-K-channel
  activation scale could not be factored out of an integer dot product over K.
* Scale: with t = fl(alpha * amax), the dequantisation scale is
  s = fl(t / qmax) and the quantisation multiplier is inv = fl(qmax / t), both
  computed once per row by IEEE division; qmax = 2^(b-1) - 1 (7 or 127),
  symmetric range [-qmax, qmax] (-8 / -128 never produced).  A row with
  t < 2^-120 (all-zero, or so small that qmax / t would overflow binary32) is
  a zero row: s = 0 and all codes 0.
* Quantise: q = clamp(rint_half_even(u * inv), -qmax, qmax) with the product
  u * inv taken exactly (it is exact in binary64 for binary32 operands) and
  rounded once, to the nearest integer.  The clip ratio is limited to
  alpha >= 2^-14, so |u * inv| <= qmax / alpha < 2^22.
* Pack: row-major, int8 as two's complement bytes; int4 as two's complement
  nibbles, element 2j in the low nibble and element 2j+1 in the high nibble of
  byte j; 6-bit codes (qmax 31, the pages' W4A6 activations) as int8 bytes.
* Integer GEMM: acc[m, n] = sum_k qa[m, k] * qw[n, k], exact (int64 here,
  checked to fit int32).
* Dequantising epilogue: out = bf16_rne(fl(fl(fl(s_a * s_w) * float(acc)) + bias)),
  bias bf16 (absent bias adds +0.0).

Every binary32 operation below is a separate numpy float32 ufunc call, so each
is one IEEE-754 round-to-nearest-even operation (numpy never contracts a*b+c
into an FMA).  Reductions used are max (exact, order free) and integer sums.
"""

from __future__ import annotations

import math

import numpy as np

QMAX = {4: 7, 6: 31, 8: 127}
# bytes of storage per code: 4-bit codes are packed two per byte; 6- and 8-bit
# codes take one byte each (6-bit codes ride in int8 containers).
STORAGE_BITS = {4: 4, 6: 8, 8: 8}
HADAMARD_BLOCK = 128
# (1/sqrt(128))^2: exact power of two carried by the weight scale.
WEIGHT_SCALE_FOLD = np.float32(2.0 ** -7)


# ---------------------------------------------------------------------------
# bf16 <-> binary32 (bit-level, no library rounding)
# ---------------------------------------------------------------------------

def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to binary32."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round binary32 to bf16, round-to-nearest, ties-to-even; returns uint16.

    Adding 0x7FFF plus the lowest kept bit and truncating is the usual RNE on
    the 16 discarded bits; overflow of the largest finite values carries into
    the exponent and correctly produces infinity.  NaN stays a quiet NaN.
    """
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    nan = np.isnan(f)
    if nan.any():
        r = r.copy()
        r[nan] = np.uint16(0x7FC0)
    return r


# ---------------------------------------------------------------------------
# Hadamard rotation (ARQ, DVD-Quant §2.B: rotate activations and weights)
# ---------------------------------------------------------------------------

def fwht128_blocks(x: np.ndarray) -> np.ndarray:
    """Unnormalised block Walsh-Hadamard transform along the last axis.

    x: binary32 [R, K] with K % 128 == 0.  Returns u = x_blk · H_128 for every
    block of 128 consecutive columns, computed by the butterfly with stages
    h = 1, 2, 4, ..., 64 in that order, one binary32 add/sub per output.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    R, K = x.shape
    if K % HADAMARD_BLOCK:
        raise ValueError("K must be a multiple of 128")
    v = x.reshape(R, K // HADAMARD_BLOCK, HADAMARD_BLOCK).copy()
    h = 1
    while h < HADAMARD_BLOCK:
        # view the block as [128 / (2h)][2][h]: index i = g*2h + half*h + j
        w = v.reshape(R, K // HADAMARD_BLOCK, HADAMARD_BLOCK // (2 * h), 2, h)
        a = w[:, :, :, 0, :].copy()
        b = w[:, :, :, 1, :].copy()
        w[:, :, :, 0, :] = a + b
        w[:, :, :, 1, :] = a - b
        h *= 2
    return v.reshape(R, K)


# ---------------------------------------------------------------------------
# Online per-token scaling and quantisation (ARQ scales from rotated values)
# ---------------------------------------------------------------------------

# Rows whose clipped absmax t is below this are zero rows (qmax / t must stay finite).
ZERO_ROW_T = np.float32(2.0 ** -120)


def row_scales(u: np.ndarray, bits: int, alpha: float) -> tuple[np.ndarray, np.ndarray]:
    """Per row of the rotated values u: (s, inv) with t = fl(alpha * amax),
    s = fl(t / qmax) (dequantisation) and inv = fl(qmax / t) (quantisation).
    Zero rows (t < 2^-120) get s = 0 and inv = 0."""
    if bits not in QMAX:
        raise ValueError("bits must be 4, 6 or 8")
    qmax = np.float32(QMAX[bits])
    amax = np.max(np.abs(u), axis=1).astype(np.float32)
    t = (np.float32(alpha) * amax).astype(np.float32)
    zero = t < ZERO_ROW_T
    safe_t = np.where(zero, np.float32(1), t).astype(np.float32)
    s = np.where(zero, np.float32(0), t / qmax).astype(np.float32)
    inv = np.where(zero, np.float32(0), qmax / safe_t).astype(np.float32)
    return s, inv


def quantize_with_scale(u: np.ndarray, inv: np.ndarray, bits: int) -> np.ndarray:
    """q = clamp(rint_half_even(u * inv), -qmax, qmax), the product exact (binary64
    holds the product of two binary32 values exactly); zero rows (inv == 0) give 0."""
    qmax = float(QMAX[bits])
    inv = np.asarray(inv, dtype=np.float32).astype(np.float64)
    r = np.asarray(u, dtype=np.float32).astype(np.float64) * inv[:, None]
    q = np.rint(r)
    q = np.minimum(np.maximum(q, -qmax), qmax)
    return q.astype(np.int8)


def quantize_rows(x_bits: np.ndarray, bits: int, alpha: float,
                  rotate: bool = True) -> tuple[np.ndarray, np.ndarray]:
    """Rotate (optionally), scale per row, quantise.  Returns (q int8 [R,K], s f32 [R]).

    x_bits: bf16 bit patterns [R, K].  ``rotate=False`` skips the Hadamard
    (used to exercise rounding ties on hand-written rows).
    """
    x = bf16_bits_to_f32(np.asarray(x_bits))
    if x.ndim != 2:
        raise ValueError("expected a 2-D array")
    if not (2.0 ** -14 <= alpha <= 1.0):
        raise ValueError("alpha must be in [2^-14, 1]")
    u = fwht128_blocks(x) if rotate else x.copy()
    s, inv = row_scales(u, bits, alpha)
    return quantize_with_scale(u, inv, bits), s


def quant_act(x_bits, bits: int, alpha: float, rotate: bool = True):
    """Activation path: per-token codes and per-token scale s_a."""
    return quantize_rows(x_bits, bits, alpha, rotate)


def pack_weights(w_bits, bits: int, rotate: bool = True):
    """Weight path (offline): per-output-channel codes, alpha = 1, and the
    channel scale s_w = fl(s * 2^-7) that carries both rotations' 1/sqrt(128)."""
    q, s = quantize_rows(w_bits, bits, 1.0, rotate)
    fold = WEIGHT_SCALE_FOLD if rotate else np.float32(1.0)
    return q, (s * fold).astype(np.float32)


# ---------------------------------------------------------------------------
# Packing
# ---------------------------------------------------------------------------

def pack(q: np.ndarray, bits: int) -> np.ndarray:
    """Pack int8 codes [R, K] to the byte layout [R, K*storage/8] (uint8)."""
    q = np.asarray(q, dtype=np.int8)
    if bits in (6, 8):
        return q.view(np.uint8).copy()
    if bits != 4:
        raise ValueError("bits must be 4, 6 or 8")
    nib = q.astype(np.uint8) & np.uint8(0x0F)
    lo = nib[:, 0::2]
    hi = nib[:, 1::2]
    return (lo | (hi << np.uint8(4))).astype(np.uint8)


def unpack(p: np.ndarray, bits: int) -> np.ndarray:
    """Inverse of :func:`pack`: bytes [R, K*bits/8] -> int8 codes [R, K]."""
    p = np.asarray(p, dtype=np.uint8)
    if bits in (6, 8):
        return p.view(np.int8).copy()
    if bits != 4:
        raise ValueError("bits must be 4, 6 or 8")
    lo = (p & np.uint8(0x0F)).astype(np.int16)
    hi = (p >> np.uint8(4)).astype(np.int16)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.int8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


# ---------------------------------------------------------------------------
# Integer GEMM and dequantising epilogue
# ---------------------------------------------------------------------------

def int_gemm(qa: np.ndarray, qw: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k qa[m, k] * qw[n, k], exact in int64."""
    a = np.asarray(qa, dtype=np.int64)
    w = np.asarray(qw, dtype=np.int64)
    acc = a @ w.T
    if acc.size and (acc.max() > 2**31 - 1 or acc.min() < -2**31):
        raise OverflowError("accumulator does not fit int32")
    return acc


def int_gemm_f64(qa: np.ndarray, qw: np.ndarray) -> np.ndarray:
    """The same accumulators through a binary64 matrix product (BLAS), for
    full-size checks where the exact int64 product is too slow.

    Exact: every code is an integer with |q| <= 127, so every partial sum that
    any summation order (or fused multiply-add) forms is an integer of
    magnitude at most sum_k |qa[m,k]| |qw[n,k]| <= 127^2 K, below 2^53 for
    every K < 5.5e11 -- binary64 represents all of them, and no rounding
    happens.  Returns int64, checked to fit int32 like :func:`int_gemm`.
    """
    a = np.asarray(qa, dtype=np.int8)
    w = np.asarray(qw, dtype=np.int8)
    if a.shape[1] * 127 * 127 >= 2 ** 53:
        raise ValueError("K too large for an exact binary64 product")
    acc = (a.astype(np.float64) @ w.astype(np.float64).T).astype(np.int64)
    if acc.size and (acc.max() > 2**31 - 1 or acc.min() < -2**31):
        raise OverflowError("accumulator does not fit int32")
    return acc


def epilogue(acc: np.ndarray, s_a: np.ndarray, s_w: np.ndarray,
             bias_bits: np.ndarray | None) -> np.ndarray:
    """out = bf16_rne(fl(fl(fl(s_a*s_w) * float(acc)) + bias)); returns uint16 bits."""
    s_a = np.asarray(s_a, dtype=np.float32)
    s_w = np.asarray(s_w, dtype=np.float32)
    sab = s_a[:, None] * s_w[None, :]
    accf = np.asarray(acc, dtype=np.int64).astype(np.int32).astype(np.float32)
    p = sab * accf
    if bias_bits is None:
        b = np.zeros(s_w.shape, dtype=np.float32)
    else:
        b = bf16_bits_to_f32(np.asarray(bias_bits))
    y = p + b[None, :]
    return f32_to_bf16_bits(y)


def qlinear(x_bits, w_bits, bias_bits, bits: int, alpha: float,
            rotate: bool = True):
    """The whole layer: quantise activations and weights, integer GEMM, dequantise.

    Returns a dict with every intermediate (codes, scales, packed bytes, acc, out).
    """
    qa, sa = quant_act(x_bits, bits, alpha, rotate)
    qw, sw = pack_weights(w_bits, bits, rotate)
    acc = int_gemm(qa, qw)
    out = epilogue(acc, sa, sw, bias_bits)
    return {"qa": qa, "sa": sa, "qw": qw, "sw": sw,
            "xp": pack(qa, bits), "wp": pack(qw, bits), "acc": acc, "out": out}


def qlinear_mixed(x_bits, w_bits, bias_bits, bits_x: int, bits_w: int, alpha: float,
                  rotate: bool = True):
    """The layer with different code widths for activations and weights
    (QuantSparse "Resumen técnico" §4: W4A8; DVD-Quant "Resumen técnico" §4: W4A6): each side is quantised at its own
    width, the integer product and the epilogue are unchanged."""
    qa, sa = quant_act(x_bits, bits_x, alpha, rotate)
    qw, sw = pack_weights(w_bits, bits_w, rotate)
    acc = int_gemm(qa, qw)
    out = epilogue(acc, sa, sw, bias_bits)
    return {"qa": qa, "sa": sa, "qw": qw, "sw": sw,
            "xp": pack(qa, bits_x), "wp": pack(qw, bits_w), "acc": acc, "out": out}


def gemm_rows(qa_rows: np.ndarray, qw: np.ndarray) -> np.ndarray:
    """Accumulators of a few activation rows against all weight rows (sampling)."""
    return int_gemm(qa_rows, qw)


# ---------------------------------------------------------------------------
# Chain glue and fp64 references
# ---------------------------------------------------------------------------

def gelu_erf_bf16(x_bits: np.ndarray) -> np.ndarray:
    """GELU with the exact erf form, x * Phi(x), evaluated in binary64 and
    rounded to bf16 (the chain's activation between ffn-up and ffn-down).
    Phi(x) = erfc(-x / sqrt(2)) / 2, the same function as (1 + erf(x/sqrt(2)))/2
    without its cancellation for x << 0."""
    x = bf16_bits_to_f32(x_bits).astype(np.float64)
    erfc = np.vectorize(math.erfc, otypes=[np.float64])
    y = 0.5 * x * erfc(-x / math.sqrt(2.0))
    return f32_to_bf16_bits(y.astype(np.float32))


def hadamard_rotation_f64(K: int) -> np.ndarray:
    """R = blockdiag(H_128) / sqrt(128) in binary64, built by Sylvester doubling."""
    h = np.array([[1.0]])
    while h.shape[0] < HADAMARD_BLOCK:
        h = np.block([[h, h], [h, -h]])
    h = h / math.sqrt(HADAMARD_BLOCK)
    r = np.zeros((K, K))
    for b in range(K // HADAMARD_BLOCK):
        sl = slice(b * HADAMARD_BLOCK, (b + 1) * HADAMARD_BLOCK)
        r[sl, sl] = h
    return r


def linear_f64(x_bits, w_bits, bias_bits=None) -> np.ndarray:
    """Unquantised x·W^T + b in binary64 from the same bf16 inputs."""
    x = bf16_bits_to_f32(x_bits).astype(np.float64)
    w = bf16_bits_to_f32(w_bits).astype(np.float64)
    y = x @ w.T
    if bias_bits is not None:
        y = y + bf16_bits_to_f32(bias_bits).astype(np.float64)[None, :]
    return y
