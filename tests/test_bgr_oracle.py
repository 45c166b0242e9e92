"""Pins of the BGR oracle (DVD-Quant "Resumen técnico" §2.A) against what the
pages and the mathematics fix, and planted mistakes that the pins catch."""

import os

import numpy as np
import pytest

import oracle.bgr_oracle as B
from oracle import qs_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "bgr_worked_w4.txt")


def _golden():
    d = {}
    with open(GOLDEN) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                k, *v = line.split()
                d[k] = v
    return d


def _gauss_rows(seed, n, k, outliers=3, factor=12.0):
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((n, k))
    for r in range(n):
        u[r, rng.choice(k, outliers, replace=False)] *= factor
    return u.astype(np.float32).astype(np.float64)


# --------------------------------------------------------------------------- pins

def pin_worked_example(b=B):
    g = _golden()
    u = np.array([float(v) for v in g["u"]])
    d, z, q, e = b.bgr_row(u, int(g["bits"][0]), int(g["candidates"][0]),
                           int(g["iterations"][0]))
    assert d == float(g["step"][0]) and z == int(g["zero"][0]) and e == float(g["error"][0])
    assert q.tolist() == [int(v) for v in g["codes"]]


def pin_exact_grid_recovered(b=B):
    """A row lying exactly on an asymmetric grid with both end levels present
    is reproduced with zero error (step, zero point and codes)."""
    rng = np.random.default_rng(4)
    for bits in (4, 8):
        levels = (1 << bits) - 1
        for z0 in (0, 3, levels // 2, levels):
            step = 2.0 ** -5
            q0 = rng.integers(0, levels + 1, 300)
            q0[:2] = (0, levels)
            u = step * (q0 - z0)
            d, z, q, e = b.bgr_row(u, bits, 16, 4)
            assert (d, z, e) == (step, z0, 0.0) and np.array_equal(q, q0), (bits, z0)


def pin_least_squares_optimality(b=B):
    """For the zero point it returns, the refit step zeroes the derivative of
    the error; on data on a line the fit recovers step and zero point."""
    u = _gauss_rows(1, 1, 640)[0]
    q = b.grid_codes(u, 0.4, 7, 4)
    d, z = b.least_squares_grid(u, q, 4)
    t = (q - z).astype(np.float64)
    assert abs(np.sum((u - d * t) * t)) <= 1e-9 * np.sum(np.abs(u * t))
    q2 = np.arange(256) % 16
    d2, z2 = b.least_squares_grid(0.125 * (q2 - 5.0), q2, 4)
    assert (d2, z2) == (0.125, 5)


def pin_codes_and_error_definition(b=B):
    """Codes stay in [0, 2^b - 1]; the error equals the brute-force loop."""
    u = _gauss_rows(2, 1, 200)[0]
    for bits, d, z in ((4, 0.3, 8), (8, 0.02, 128), (4, 1e-3, 0)):
        q = b.grid_codes(u, d, z, bits)
        assert q.min() >= 0 and q.max() <= (1 << bits) - 1
        acc = 0.0
        for k in range(u.size):
            e = float(u[k]) - d * float(q[k] - z)
            acc = acc + e * e
        assert b.grid_error(u, d, z, q) == acc


def pin_refinement_never_worse_and_beats_minmax(b=B):
    """The kept grid is never worse than the MinMax grid or the bound search,
    and on Gaussian rows with outliers it is clearly better than MinMax (the
    pages' motivation)."""
    u = _gauss_rows(3, 24, 512)
    for bits in (4, 8):
        ratios, refined = [], 0
        for row in u:
            d0, z0 = b.grid_from_bounds(row.min(), row.max(), bits)
            e0 = b.grid_error(row, d0, z0, b.grid_codes(row, d0, z0, bits))
            _, _, es = b.bound_search(row, bits, 32)
            _, _, _, e = b.bgr_row(row, bits, 32, 6)
            assert e <= es <= e0
            ratios.append(e / e0)
            refined += e < es
        assert refined >= len(u) // 4, (bits, refined)  # the refits improve on the search
        # 16 levels: clipping the rare outliers pays; 256 levels: MinMax is
        # already close to the best grid
        if bits == 4:
            assert np.median(ratios) < 0.85, np.median(ratios)


def pin_asymmetric_accumulators_bruteforce(b=B):
    """acc = sum qa (s + o) = sum qa (q - z) on a small layer, by loops."""
    rng = np.random.default_rng(8)
    x = O.f32_to_bf16_bits(rng.standard_normal((5, 128)).astype(np.float32))
    w = O.f32_to_bf16_bits((rng.standard_normal((6, 128)) * 0.02).astype(np.float32))
    for bits in (4, 8):
        r = b.qlinear_bgr(x, w, None, bits, 1.0, 8, 2)
        half = 1 << (bits - 1)
        assert r["s"].min() >= -half and r["s"].max() <= half - 1
        for m in range(5):
            for n in range(6):
                z = half - int(r["offset"][n])
                want = sum(int(r["qa"][m, k]) * (int(r["s"][n, k]) + half - z) for k in range(128))
                assert int(r["acc"][m, n]) == want


def pin_layer_error_not_worse_than_symmetric(b=B):
    """Through the rotated layer, BGR weights give a smaller output error than
    the symmetric per-channel weights on weights with outlier entries."""
    rng = np.random.default_rng(9)
    x = O.f32_to_bf16_bits(rng.standard_normal((64, 256)).astype(np.float32))
    wf = rng.standard_normal((48, 256)) * 0.02
    wf[:, rng.choice(256, 4, replace=False)] *= 20
    w = O.f32_to_bf16_bits(wf.astype(np.float32))
    ref = O.linear_f64(x, w)
    for bits in (4, 8):
        sym = O.bf16_bits_to_f32(O.qlinear(x, w, None, bits, 1.0)["out"]).astype(np.float64)
        bgr = O.bf16_bits_to_f32(b.qlinear_bgr(x, w, None, bits, 1.0)["out"]).astype(np.float64)
        assert np.linalg.norm(bgr - ref) < np.linalg.norm(sym - ref), bits


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


# --------------------------------------------------------------------------- mutants

def _error_abs(u, delta, z, q):
    dq = np.float64(delta) * (q - z).astype(np.float64)
    return B.seq_sum(np.abs(np.asarray(u, np.float64) - dq))


def _symmetric_grid(lo, hi, bits):
    levels = (1 << bits) - 1
    return float((np.float64(hi) - np.float64(lo)) / levels), 1 << (bits - 1)


def _codes_truncated(u, delta, z, bits):
    r = np.trunc(np.asarray(u, np.float64) * (1.0 / delta))
    return np.clip(r + z, 0, (1 << bits) - 1).astype(np.int64)


def _accum_offset_negated(qa, s, offset):
    return O.int_gemm(qa, s) - B.code_rowsums(qa)[:, None] * np.asarray(offset, np.int64)[None, :]


MUTANTS = {
    "absolute_error": ("grid_error", _error_abs),
    "zero_point_fixed_at_half": ("grid_from_bounds", _symmetric_grid),
    "codes_truncated": ("grid_codes", _codes_truncated),
    "offset_sign_flipped": ("asym_accumulators", _accum_offset_negated),
    "no_refinement": ("least_squares_grid", lambda u, q, bits: None),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(B, attr, fn)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(B)
        except Exception as e:  # noqa: BLE001 - any failure of a pin counts
            caught.append((pin.__name__, type(e).__name__))
    assert caught, f"no pin catches the mutant {name}"
