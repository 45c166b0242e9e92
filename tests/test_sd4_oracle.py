"""Pins of the SD4 oracle (SemanticDialect "Resumen técnico" §2.A) against the
mathematics of its construction (parity against the pages is unpinned: they
print no formatbook), and planted mistakes that the pins catch."""

import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle.sd4_oracle as S
from oracle import qs_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "sd4_formatbook_rows.txt")


def _bf16(x):
    return O.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _rows(seed, r, k, outliers=2):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((r, k))
    for i in range(r):
        x[i, rng.choice(k, outliers, replace=False)] *= 15
    return _bf16(x)


def pin_formatbook_rows_and_shape(s=S):
    L = s.formatbook()
    with open(GOLDEN) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                d, *lv = (int(v) for v in line.split())
                assert L[d].tolist() == lv, d
    assert L.shape == (32, 8) and len({tuple(r) for r in L.tolist()}) == 32
    assert (L[:, 0] == 0).all() and (np.diff(L, axis=1) > 0).all()
    assert sorted(set(L[:, 7].tolist())) == [12, 13, 14, 15]


def pin_lut_is_the_nearest_level(s=S):
    """Qvalue is the nearest level of every value in the bin (exact rationals,
    values at both bin edges and inside), and Qerror the bin centre's squared
    distance to it."""
    L = s.formatbook()
    qerr, qval = s.lut_tables(L)
    for d in (0, 5, 13, 31):
        for b in range(256):
            lo, hi = Fraction(b, 128), Fraction(b + 1, 128)
            for v in (lo, (lo + hi) / 2, hi - Fraction(1, 1 << 20)):
                dist = [abs(v - Fraction(int(l), 8)) for l in L[d]]
                best = min(dist)
                assert dist[qval[d, b]] == best, (d, b, v)
            c = Fraction(2 * b + 1, 256)
            assert qerr[d, b] == min((c - Fraction(int(l), 8)) ** 2 for l in L[d]) * 65536


def pin_qvalue_changes_only_at_multiples_of_eight_bins(s=S):
    """Levels are multiples of 1/8 and bins 1/128 wide, so every midpoint
    (L_i + L_i+1)/16 between neighbouring levels falls on a multiple of 8
    bins: Qvalue is constant on each run of 8 bins, and it steps exactly at
    bin 8 (L_i + L_i+1) for every pair of levels of the dialect."""
    L = s.formatbook()
    _, qval = s.lut_tables(L)
    for d in range(32):
        assert np.array_equal(qval[d], np.repeat(qval[d, ::8], 8)), d
        steps = sorted(set(int(8 * (L[d, i] + L[d, i + 1])) for i in range(7)))
        got = [b for b in range(1, 256) if qval[d, b] != qval[d, b - 1]]
        assert got == [t for t in steps if t < 256], (d, got, steps)


def pin_block_scale(s=S):
    """amax normalises into [1, 2); zero blocks; the floor at 2^-126."""
    for amax in (1.0, 1.999, 2.0, 0.75, 3e-5, 6e4):
        e = s.block_exponent(amax)
        assert 1.0 <= amax * 2.0 ** -e < 2.0, amax
    assert s.block_exponent(0.0) == 0
    assert s.block_exponent(2.0 ** -130) == -126


def pin_codes_are_nearest_levels_of_the_best_dialect(s=S):
    """Every decoded value is the chosen dialect's nearest level (brute force),
    and the chosen dialect minimises the table cost (brute force over 32)."""
    x = _rows(4, 6, 256)
    codes, exps, dias = s.quantize_rows(x)
    L = s.formatbook()
    qerr, _ = s.lut_tables(L)
    xf = O.bf16_bits_to_f32(x).astype(np.float64)
    xh = s.dequantize(codes, exps, dias)
    for r in range(6):
        for j in range(8):
            blk = xf[r, 32 * j:32 * j + 32]
            e, d = int(exps[r, j]), int(dias[r, j])
            amax = float(np.max(np.abs(blk)))
            assert amax == 0 or 1.0 <= amax * 2.0 ** -e < 2.0
            bins = [min(int(math.floor(abs(v) * 2.0 ** -e * 128)), 255) for v in blk]
            costs = [sum(int(qerr[dd, b]) for b in bins) for dd in range(32)]
            assert d == costs.index(min(costs))
            for k in range(32):
                levels = [int(l) / 8 * 2.0 ** e for l in L[d]]
                dist = [abs(abs(blk[k]) - lv) for lv in levels]
                got = abs(xh[r, 32 * j + k])
                assert abs(abs(blk[k]) - got) == min(dist)
                assert (xh[r, 32 * j + k] < 0) == (blk[k] < 0) or got == 0


def pin_zero_and_exact_blocks(s=S):
    """An all-zero block decodes to zeros; a block whose values are one
    dialect's levels decodes exactly (the levels are in the bins' nearest set)."""
    L = s.formatbook()
    x = np.zeros((2, 64), np.float32)
    x[1, :8] = L[5] / 8 * 4.0
    x[1, 8:16] = -L[5] / 8 * 4.0
    x[1, 16:32] = 15 / 8 * 4.0
    codes, exps, dias = s.quantize_rows(_bf16(x))
    xh = s.dequantize(codes, exps, dias)
    assert not xh[0].any() and not xh[1, 32:].any()
    # every value is a level of dialect 5 (bin centre 1/256 above it: cost 32);
    # a dialect lacking one of them costs more, so 5 is chosen and decodes exactly
    assert int(dias[1, 0]) == 5 and int(exps[1, 0]) == 2
    assert np.array_equal(xh[1, :32], x[1, :32].astype(np.float64))


def pin_mixed_formats_beat_a_fixed_format(s=S):
    """Per-block dialect choice gives a smaller error than the uniform dialect
    (d = 0) everywhere (the pages' motivation for mixed formats)."""
    x = _rows(7, 16, 512)
    xf = O.bf16_bits_to_f32(x).astype(np.float64)
    codes, exps, dias = s.quantize_rows(x)
    e_mixed = np.sum((s.dequantize(codes, exps, dias) - xf) ** 2)
    qerr, qval = s.lut_tables()
    fixed = np.zeros_like(codes)
    for r in range(16):
        for j in range(16):
            e = int(exps[r, j])
            blk = xf[r, 32 * j:32 * j + 32]
            bins = np.minimum(np.floor(np.abs(blk) * 2.0 ** -e * 128), 255).astype(int)
            fixed[r, 32 * j:32 * j + 32] = ((blk < 0) << 3) | qval[0, bins]
    e_fixed = np.sum((s.dequantize(fixed, exps, np.zeros_like(dias)) - xf) ** 2)
    assert e_mixed < 0.9 * e_fixed, (e_mixed, e_fixed)


def pin_layer_exact_sum(s=S):
    """The layer's accumulator is the exact sum of decoded products (brute
    force) and the output its binary32 value plus the bias, in bf16."""
    x, w = _rows(1, 3, 64), _rows(2, 4, 64)
    b = _bf16(np.array([0.5, -1.0, 0.0, 2.0]))
    r = s.linear_sd4(x, w, b)
    for m in range(3):
        for n in range(4):
            exact = sum(Fraction(float(r["x_hat"][m, k])) * Fraction(float(r["w_hat"][n, k]))
                        for k in range(64))
            assert r["y"][m, n] == float(exact)
            want = O.f32_to_bf16_bits(np.float32(np.float32(float(exact)) +
                                                  O.bf16_bits_to_f32(b)[n]))
            assert r["out"][m, n] == want


def _check_nearest_levels(s, vals, dec, exps, dias):
    """Brute force: every block's dialect minimises the table cost over the 32
    dialects and every value `dec` (what the layer uses) is that dialect's
    nearest level (signed)."""
    L = s.formatbook()
    qerr, _ = s.lut_tables(L)
    R, K = vals.shape
    for r in range(R):
        for j in range(K // 32):
            blk = vals[r, 32 * j:32 * j + 32]
            e, d = int(exps[r, j]), int(dias[r, j])
            amax = float(np.max(np.abs(blk)))
            assert amax == 0 or 1.0 <= amax * 2.0 ** -e < 2.0
            bins = [min(int(math.floor(abs(v) * 2.0 ** -e * 128)), 255) for v in blk]
            costs = [sum(int(qerr[dd, b]) for b in bins) for dd in range(32)]
            assert d == costs.index(min(costs))
            levels = [int(l) / 8 * 2.0 ** e for l in L[d]]
            for k in range(32):
                got = dec[r, 32 * j + k]
                assert abs(got) in levels
                assert abs(abs(blk[k]) - abs(got)) == min(abs(abs(blk[k]) - lv) for lv in levels)
                assert got == 0 or (got < 0) == (blk[k] < 0)


def _two_scale_rows(seed, R, K, d_res=13):
    """Rows of blocks x = a + b: a in {0, +-15/8} 2^e, b = +-L/8 2^(e-4) with L
    levels of dialect d_res (its top level in every block) where a != 0, else 0.
    x is bf16-exact ((240 +- L) 2^(e-7)); Q(A) = a (15/8 is the nearest level in
    every dialect whose top level is 15, and those dialects cost least);
    Delta = b has block exponent e-4 and is exactly one dialect's levels."""
    rng = np.random.default_rng(seed)
    L = S.formatbook()
    x = np.zeros((R, K))
    a_all = np.zeros((R, K))
    for r in range(R):
        for j in range(K // 32):
            e = int(rng.integers(-20, 20))
            nz = rng.choice(32, 20, replace=False)
            a = np.zeros(32)
            a[nz] = rng.choice([-1.0, 1.0], 20) * 15 / 8 * 2.0 ** e
            b = np.zeros(32)
            idx = rng.integers(0, 8, 20)
            idx[0] = 7
            b[nz] = rng.choice([-1.0, 1.0], 20) * L[d_res, idx] / 8 * 2.0 ** (e - 4)
            x[r, 32 * j:32 * j + 32] = a + b
            a_all[r, 32 * j:32 * j + 32] = a
    bits = _bf16(x)
    assert np.array_equal(O.bf16_bits_to_f32(bits).astype(np.float64), x)
    return bits, x, a_all


def pin_decomposition_residual_is_exact_and_requantised(s=S):
    """Delta = A - x_hat exactly (a binary32 number); Q(A) of the salient rows
    is the plain quantisation; Q(Delta) is a nearest-level SD4 quantisation of
    Delta (brute force); the residual step moves no element away from A (level
    0 is in every dialect) and cuts the total error."""
    x = _rows(11, 5, 256, outliers=4)
    rows = [4, 0, 2, 2]
    dec = s.decompose_rows(x, rows)
    xf = O.bf16_bits_to_f32(x).astype(np.float64)[rows]
    assert np.array_equal(dec["x_hat"] + dec["delta"], xf)
    assert np.array_equal(dec["delta"].astype(np.float32).astype(np.float64), dec["delta"])
    _check_nearest_levels(s, xf, dec["x_hat"], dec["exp_x"], dec["dia_x"])
    _check_nearest_levels(s, dec["delta"], dec["d_hat"], dec["exp_d"], dec["dia_d"])
    assert np.array_equal(s.dequantize(dec["codes_d"], dec["exp_d"], dec["dia_d"]), dec["d_hat"])
    err0 = np.abs(xf - dec["x_hat"])
    err1 = np.abs(xf - dec["x_hat"] - dec["d_hat"])
    assert (err1 <= err0).all() and err1.sum() < 0.5 * err0.sum()


def pin_decomposition_reconstructs_two_scale_blocks(s=S):
    """On blocks that are a sum of levels at two scales, Q(A) is the coarse
    part and Q(Delta) the fine part, so x_hat + delta_hat = A exactly."""
    bits, x, a = _two_scale_rows(5, 3, 256)
    dec = s.decompose_rows(bits, [0, 1, 2])
    assert np.array_equal(dec["x_hat"], a)
    assert np.array_equal(dec["x_hat"] + dec["d_hat"], x)


def pin_decomposed_layer(s=S):
    """No salient rows: the plain layer.  Two-scale rows (reconstructed
    exactly) as the salient rows: their accumulators are the exact products of
    A itself with w_hat (brute force), the other rows keep x_hat's."""
    bits, x, _ = _two_scale_rows(9, 4, 64)
    w = _rows(3, 3, 64)
    b = _bf16(np.array([0.25, -1.0, 0.0]))
    plain = s.linear_sd4(bits, w, b)
    r0 = s.linear_sd4_decomp(bits, w, b, [])
    assert np.array_equal(r0["out"], plain["out"])
    r = s.linear_sd4_decomp(bits, w, b, [2, 0])
    bf = O.bf16_bits_to_f32(b)
    for m in range(4):
        for n in range(3):
            src = x[m] if m in (0, 2) else plain["x_hat"][m]
            exact = sum(Fraction(float(src[k])) * Fraction(float(r["w_hat"][n, k]))
                        for k in range(64))
            assert r["y"][m, n] == float(exact)
            assert r["out"][m, n] == O.f32_to_bf16_bits(np.float32(np.float32(float(exact)) + bf[n]))


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


# --------------------------------------------------------------------------- mutants

def _lut_half_scale(L=None):
    L = S.formatbook() if L is None else L
    b = np.arange(256)[None, :, None]
    dist = (2 * b + 1 - 16 * L[:, None, :]) ** 2
    return dist.min(axis=2), dist.argmin(axis=2)


def _exponent_ceil(amax):
    return 0 if amax == 0 else max(math.frexp(amax)[1], -126)


def _formatbook_no_raise():
    L = np.zeros((32, 8), np.int64)
    for a in range(4):
        t = 15 - a
        for sh, (p, q, r) in enumerate(S.SD4_SHAPES):
            for i in range(1, 8):
                L[8 * a + sh, i] = (2 * t * (49 * p * i + 7 * q * i * i + r * i ** 3) + 2744) // 5488
    return L


def _decompose_with(residual):
    def decompose(x_bits, rows):
        x = O.bf16_bits_to_f32(np.asarray(x_bits)).astype(np.float64)[np.asarray(rows, np.int64)]
        cx, ex, dx = S.quantize_values(x)
        x_hat = S.dequantize(cx, ex, dx)
        delta = residual(x, x_hat)
        cd, ed, dd = S.quantize_values(delta)
        d_hat = S.dequantize(cd, ed, dd) if residual is not _unquantised else delta
        return {"codes_x": cx, "exp_x": ex, "dia_x": dx, "x_hat": x_hat, "delta": delta,
                "codes_d": cd, "exp_d": ed, "dia_d": dd, "d_hat": d_hat}
    return decompose


def _unquantised(x, x_hat):
    return x - x_hat


MUTANTS = {
    "residual_sign_flipped": ("decompose_rows", _decompose_with(lambda x, xh: xh - x)),
    "residual_of_the_input": ("decompose_rows", _decompose_with(lambda x, xh: x)),
    "residual_left_unquantised": ("decompose_rows", _decompose_with(_unquantised)),
    "lut_levels_in_sixteenths": ("lut_tables", _lut_half_scale),
    "exponent_rounded_up": ("block_exponent", _exponent_ceil),
    "levels_not_strictly_increasing": ("formatbook", _formatbook_no_raise),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(S, attr, fn)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(S)
        except Exception as e:  # noqa: BLE001 - any failure of a pin counts
            caught.append((pin.__name__, type(e).__name__))
    assert caught, f"no pin catches the mutant {name}"
