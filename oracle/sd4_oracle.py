"""CPU oracle of the SD4 block format (SemanticDialect's mixed-format 4-bit
quantisation) for the linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only the test-suite, the smoke check and the CPU-baseline
leg of the benchmark use it.  It shares no code with the CUDA library.

What the pages fix (SemanticDialect, "Resumen técnico" §2.A, "Cuantización
Mixta de Formato por Bloque (SD4)", and §3 item 1): a formatbook of 32
candidate 4-bit "dialects", each a set of representable values; every small
block of activations or weights uses the dialect that fits its values best;
the choice and the quantisation use precomputed tables (Qvalue, Qerror); each
block shares a power-of-two scale that normalises its values to [0, 2), which
are then mapped to 4-bit integers.  Block size 32 is the one the results
mention (§4).

PARITY UNPINNED against the pages: they print no dialect table, so the
formatbook below is this implementation's own (a reading), and the pins check
the construction against the mathematics, not against the paper's values.

Readings:

* Code: 1 sign bit (bit 3) + a 3-bit level index i; the dialect d maps i to
  the magnitude L[d][i] / 8 with integer L, L[d][0] = 0 (so every dialect has
  0 and 7 nonzero magnitudes below 2).
* Formatbook, d = 8 a + s (a = 0..3, s = 0..7): top level t = 15 - a and the
  shape s, a blend (p, q, r)/8 of the ramp i/7, its square and its cube:
  (8,0,0) (6,2,0) (4,4,0) (3,5,0) (2,5,1) (0,8,0) (1,3,4) (0,3,5), from
  uniform levels to levels crowded near zero.  For i = 1..7,
  L = floor((2 t (49 p i + 7 q i^2 + r i^3) + 2744) / 5488) -- the integer
  nearest (half up) to t (p i/7 + q (i/7)^2 + r (i/7)^3) / 8 -- then made
  strictly increasing (L[i] = max(L[i], L[i-1] + 1)).  L[d][7] = t always, and
  the 32 level sets are distinct.
* Block scale: e = max(floor(log2 amax), -126) over the 32 elements of the
  block (e = 0 for an all-zero block); normalised magnitude v = |x| 2^-e,
  which lies in [0, 2).
* Bins: b = min(floor(128 v), 255).  Qerror[d][b] = min_i (2b + 1 - 32 L[d][i])^2
  (an integer: the squared distance, in units of 2^-8, from the bin centre to
  the dialect's nearest level); Qvalue[d][b] = that nearest i (never a tie:
  2b + 1 is odd, 32 L even).  Level midpoints are multiples of 1/16, i.e.
  bin edges, so Qvalue is the exact nearest level of every value in the bin
  (a value exactly on a midpoint goes to the upper level).
* Dialect of a block: argmin_d sum_k Qerror[d][b_k] (exact integer sums; the
  smallest d on ties).
* Element code: (x < 0) << 3 | Qvalue[d][b]; decoded value (-1)^s L/8 2^e, which
  is exact in binary32 and in bf16.
* Storage: codes two per byte (element 2j in the low nibble of byte j), one
  16-bit word per block: the low byte is e as int8, the high byte d.
* Layer: y = sum_k x_hat[m,k] w_hat[n,k] exactly, rounded to binary64 and
  then to binary32, out = bf16_rne(fl(y + bias)).  The tensor-core path accumulates in binary32,
  so the device result is compared within a bound derived in the tests.

Activation decomposition ("Resumen técnico" §2.B): a salient row A is split
into its SD4 value Q(A) and the residual Delta = A - deq(Q(A)); Delta is
quantised again with the same format and the layer uses A ~ Q(A) + Q(Delta).
Readings: Delta is the exact difference (it is a binary32 number: see
decompose_rows); its SD4 blocks are the same 32 columns as A's; the salient
rows are given by the caller (the pages pick them from attention scores of a
trained model, which this library does not have); their output is
bf16_rne(fl(sum_k (x_hat + delta_hat)[m,k] w_hat[n,k] + bias)) with the exact
sum, and the other rows are those of the plain layer.
"""

from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

from .qs_oracle import bf16_bits_to_f32, f32_to_bf16_bits

SD4_BLOCK = 32
SD4_DIALECTS = 32
SD4_BINS = 256


SD4_SHAPES = ((8, 0, 0), (6, 2, 0), (4, 4, 0), (3, 5, 0), (2, 5, 1), (0, 8, 0), (1, 3, 4),
              (0, 3, 5))


def formatbook() -> np.ndarray:
    """L[d][i], int, shape [32, 8]."""
    L = np.zeros((SD4_DIALECTS, 8), np.int64)
    for a in range(4):
        t = 15 - a
        for s, (p, q, r) in enumerate(SD4_SHAPES):
            d = 8 * a + s
            for i in range(1, 8):
                v = (2 * t * (49 * p * i + 7 * q * i * i + r * i ** 3) + 2744) // 5488
                L[d, i] = max(v, L[d, i - 1] + 1)
    return L


def lut_tables(L: np.ndarray | None = None) -> tuple[np.ndarray, np.ndarray]:
    """(Qerror[d][b], Qvalue[d][b]) for b in 0..255."""
    L = formatbook() if L is None else L
    b = np.arange(SD4_BINS)[None, :, None]
    dist = (2 * b + 1 - 32 * L[:, None, :]) ** 2          # [d, b, i]
    return dist.min(axis=2), dist.argmin(axis=2)


def block_exponent(amax: float) -> int:
    if amax == 0.0:
        return 0
    _, E = math.frexp(amax)        # amax = m 2^E, m in [0.5, 1)
    return max(E - 1, -126)


def quantize_rows(x_bits: np.ndarray):
    """SD4 codes [R, K] (uint8 nibbles 0..15), exponents [R, K/32] (int),
    dialects [R, K/32] (int)."""
    return quantize_values(bf16_bits_to_f32(np.asarray(x_bits)).astype(np.float64))


def quantize_values(x: np.ndarray):
    """quantize_rows on binary64 values (each exactly a binary32 number, as the
    residuals of the activation decomposition are)."""
    x = np.asarray(x, np.float64)
    R, K = x.shape
    if K % SD4_BLOCK:
        raise ValueError("K must be a multiple of 32")
    L = formatbook()
    qerr, qval = lut_tables(L)
    nb = K // SD4_BLOCK
    codes = np.zeros((R, K), np.uint8)
    exps = np.zeros((R, nb), np.int64)
    dias = np.zeros((R, nb), np.int64)
    for r in range(R):
        for j in range(nb):
            blk = x[r, j * SD4_BLOCK:(j + 1) * SD4_BLOCK]
            e = block_exponent(float(np.max(np.abs(blk))))
            v = np.abs(blk) * 2.0 ** (-e)                      # exact
            bins = np.minimum(np.floor(v * 128.0), 255).astype(np.int64)
            cost = qerr[:, bins].sum(axis=1)                   # exact integers
            d = int(np.argmin(cost))                           # first minimum
            idx = qval[d, bins]
            sign = (blk < 0).astype(np.uint8)
            codes[r, j * SD4_BLOCK:(j + 1) * SD4_BLOCK] = (sign << 3) | idx.astype(np.uint8)
            exps[r, j], dias[r, j] = e, d
    return codes, exps, dias


def dequantize(codes, exps, dias) -> np.ndarray:
    """Decoded values (binary64, exact) [R, K]."""
    L = formatbook()
    codes = np.asarray(codes)
    R, K = codes.shape
    d = np.repeat(np.asarray(dias), SD4_BLOCK, axis=1)
    e = np.repeat(np.asarray(exps), SD4_BLOCK, axis=1)
    mag = L[d, codes & 7].astype(np.float64) / 8.0 * np.exp2(e.astype(np.float64))
    return np.where(codes & 8, -mag, mag)


def pack_codes(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << np.uint8(4))).astype(np.uint8)


def pack_meta(exps, dias) -> np.ndarray:
    """One uint16 per block: low byte e (int8), high byte d."""
    e = (np.asarray(exps, np.int64) & 0xFF).astype(np.uint16)
    return e | (np.asarray(dias, np.uint16) << np.uint16(8))


def exact_products(xh: np.ndarray, wh: np.ndarray) -> list[list[Fraction]]:
    """sum_k x_hat w_hat exactly (rationals), for small cases."""
    M, N = xh.shape[0], wh.shape[0]
    fx = [[Fraction(float(v)) for v in row] for row in xh]
    fw = [[Fraction(float(v)) for v in row] for row in wh]
    return [[sum((a * b for a, b in zip(fx[m], fw[n])), Fraction(0)) for n in range(N)]
            for m in range(M)]


def linear_sd4(x_bits, w_bits, bias_bits=None, exact: bool = True):
    """The SD4 layer.  `exact`: the products summed exactly (rationals, small
    cases); otherwise with binary64 (error far below one binary32 rounding for
    the sizes used, stated by the tests)."""
    cx, ex, dx = quantize_rows(x_bits)
    cw, ew, dw = quantize_rows(w_bits)
    xh, wh = dequantize(cx, ex, dx), dequantize(cw, ew, dw)
    y, out = layer_outputs(xh, wh, bias_bits, exact)
    return {"codes_x": cx, "exp_x": ex, "dia_x": dx, "codes_w": cw, "exp_w": ew, "dia_w": dw,
            "x_hat": xh, "w_hat": wh, "y": y, "out": out}


def layer_outputs(x_hat, w_hat, bias_bits=None, exact: bool = True):
    """The layer's last steps on decoded operands: y = sum_k x_hat w_hat (exact
    rationals, or binary64 when not `exact`) and out = bf16_rne(fl(fl32(y) +
    bias)) as bf16 bits."""
    N = w_hat.shape[0]
    if len(x_hat) == 0:
        y = np.zeros((0, N))
    elif exact:
        y = np.array([[float(v) for v in row] for row in exact_products(x_hat, w_hat)])
    else:
        y = x_hat @ w_hat.T
    b = (np.zeros(N, np.float32) if bias_bits is None
         else bf16_bits_to_f32(np.asarray(bias_bits)))
    return y, f32_to_bf16_bits((y.astype(np.float32) + b[None, :]).astype(np.float32))


def decompose_rows(x_bits, rows):
    """Q(A) and Q(Delta) of the rows `rows` of x (bf16 bits [M, K]).

    Delta = A - x_hat is exact in binary64 and is a binary32 number: a nonzero
    x_hat is a multiple of 2^(e-3) with |x_hat| < 2^(e+1), and an element that
    rounds to a nonzero level has |A| >= 2^(e-4), so A is a multiple of
    2^(e-11) and |Delta| < 2^(e+2) spans at most 13 bits; an element that
    rounds to level 0 has Delta = A."""
    x = bf16_bits_to_f32(np.asarray(x_bits)).astype(np.float64)[np.asarray(rows, np.int64)]
    cx, ex, dx = quantize_values(x)
    x_hat = dequantize(cx, ex, dx)
    delta = x - x_hat
    cd, ed, dd = quantize_values(delta)
    return {"codes_x": cx, "exp_x": ex, "dia_x": dx, "x_hat": x_hat, "delta": delta,
            "codes_d": cd, "exp_d": ed, "dia_d": dd, "d_hat": dequantize(cd, ed, dd)}


def pack_decomp(dec) -> tuple[np.ndarray, np.ndarray]:
    """The decomposed rows as rows of 2K codes: [Q(A) | Q(Delta)] (codes two
    per byte, one block word per 32 codes)."""
    codes = np.concatenate([dec["codes_x"], dec["codes_d"]], axis=1)
    exps = np.concatenate([dec["exp_x"], dec["exp_d"]], axis=1)
    dias = np.concatenate([dec["dia_x"], dec["dia_d"]], axis=1)
    return pack_codes(codes), pack_meta(exps, dias)


def linear_sd4_decomp(x_bits, w_bits, bias_bits, rows, exact: bool = True):
    """The SD4 layer with the salient rows `rows` decomposed: those rows use
    x_hat + delta_hat (the element sum is exact in binary64), the others are
    linear_sd4's."""
    r = linear_sd4(x_bits, w_bits, bias_bits, exact=exact)
    rows = np.asarray(rows, np.int64)
    dec = decompose_rows(x_bits, rows)
    xt = dec["x_hat"] + dec["d_hat"]
    y, o = layer_outputs(xt, r["w_hat"], bias_bits, exact)
    out = r["out"].copy()
    yrows = r["y"].copy()
    if len(rows):
        out[rows] = o
        yrows[rows] = y
    r.update({"decomp": dec, "out": out, "y": yrows, "x_tilde": xt, "rows": rows})
    return r
