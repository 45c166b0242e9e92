"""Pins of the δ-GBS oracle (DVD-Quant "Resumen técnico" §2.C) against what
the pages and the mathematics fix, and planted mistakes that the pins catch."""

import math
import os
from dataclasses import dataclass
from fractions import Fraction

import numpy as np
import pytest

import oracle.gbs_oracle as G
from oracle import qs_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "gbs_decisions.txt")


def _bf16(x):
    return O.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _load_golden():
    delta, rows, widths = None, [], None
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if parts[0] == "delta":
                delta = float(parts[1])
            elif parts[0] == "widths":
                widths = [int(v) for v in parts[1:]]
            else:
                step, d, acc, nxt = parts
                rows.append((int(step), None if d == "-" else float(d), float(acc), int(nxt)))
    return delta, rows, widths


# --------------------------------------------------------------------------- pins

def pin_golden_decisions(g=G):
    """Every accumulator value and width of the hand-worked sequence."""
    delta, rows, widths = _load_golden()
    s = g.GbsState()
    assert s.bits == 8
    for step, d, acc, nxt in rows:
        s = g.gbs_update(s, d, delta)
        assert s.acc == acc and s.bits == nxt, (step, s)
    assert g.gbs_schedule([d for _, d, _, _ in rows[1:]], delta) == widths


def pin_distance_closed_forms(g=G):
    """d(y, y) = 0, d(2y, y) = 1, d(-y, y) = 2, d(0, y) = 1 (bf16 doubling and
    negation are exact); zero previous output: 0 if unchanged, else +inf."""
    rng = np.random.default_rng(3)
    y = _bf16(rng.standard_normal((7, 33)))
    y2 = _bf16(2 * O.bf16_bits_to_f32(y))
    yn = _bf16(-O.bf16_bits_to_f32(y))
    z = np.zeros_like(y)
    assert g.l1_distance(y, y) == 0.0
    assert g.l1_distance(y2, y) == 1.0
    assert g.l1_distance(yn, y) == 2.0
    assert g.l1_distance(z, y) == 1.0
    assert g.l1_distance(z, z) == 0.0
    assert g.l1_distance(y, z) == math.inf


def pin_distance_exact_rational(g=G):
    """Brute force in exact rationals: the distance is the quotient of the
    correctly rounded sums (within the one rounding of the division)."""
    rng = np.random.default_rng(11)
    for trial in range(4):
        scale = [1.0, 1e-3, 1e4, 1.0][trial]
        a = _bf16(rng.standard_normal(200) * scale)
        b = _bf16(rng.standard_normal(200) * scale * (0.5 + trial))
        fa = [Fraction(float(v)) for v in O.bf16_bits_to_f32(a)]
        fb = [Fraction(float(v)) for v in O.bf16_bits_to_f32(b)]
        num = sum(abs(x - y) for x, y in zip(fa, fb))
        den = sum(abs(y) for y in fb)
        want = float(num) / float(den)
        got = g.l1_distance(a, b)
        assert got == want
        assert abs(Fraction(got) - num / den) <= Fraction(num / den) * Fraction(3, 2 ** 53)


def pin_distance_power_of_two_scaling(g=G):
    """Scaling both outputs by 2^k changes nothing (exact in bf16 and binary64)."""
    rng = np.random.default_rng(5)
    a = _bf16(rng.standard_normal(500))
    b = _bf16(rng.standard_normal(500))
    d = g.l1_distance(a, b)
    for k in (-20, -1, 3, 40):
        sa = _bf16(O.bf16_bits_to_f32(a) * np.float32(2.0 ** k))
        sb = _bf16(O.bf16_bits_to_f32(b) * np.float32(2.0 ** k))
        assert g.l1_distance(sa, sb) == d


def pin_constant_change_period(g=G):
    """With a constant change d per step the layer returns to 8 bits every
    ceil(delta / d) measured steps."""
    for d, delta in ((0.125, 0.375), (0.25, 1.0), (0.5, 0.25), (1.0, 1.0)):
        widths = g.gbs_schedule([d] * 40, delta)
        period = math.ceil(delta / d)
        eights = [t for t, b in enumerate(widths) if b == 8]
        assert eights[0] == 0
        assert all(b - a == period + (1 if i == 0 else 0) for i, (a, b) in
                   enumerate(zip(eights, eights[1:]))), (d, delta, eights)


def pin_run_uses_previous_decision(g=G):
    """gbs_run: step 0 at 8 bits; identical inputs give d = 0, so every later
    step stays at 4 bits; each output is the layer at the width of its step."""
    rng = np.random.default_rng(2)
    x = _bf16(rng.standard_normal((5, 256)))
    w = _bf16(rng.standard_normal((16, 256)) * 0.02)
    b = _bf16(rng.standard_normal(16) * 0.01)
    r = g.gbs_run([x, x, x], w, b, 1.0, 0.5)
    assert r["bits"] == [8, 4, 4]
    assert r["d"][0] is None and r["d"][2] == 0.0
    for y, bits in zip(r["out"], r["bits"]):
        assert np.array_equal(y, O.qlinear(x, w, b, bits, 1.0)["out"])
    x2 = _bf16(O.bf16_bits_to_f32(x) * 8)  # a large change forces 8 bits next
    r = g.gbs_run([x, x, x2, x2], w, b, 1.0, 0.5)
    assert r["bits"] == [8, 4, 4, 8]


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


# --------------------------------------------------------------------------- mutants

def _distance_by_current(cur, prev):
    diff, _ = G.l1_terms(cur, prev)
    _, ref = G.l1_terms(prev, cur)
    num, den = math.fsum(diff.tolist()), math.fsum(ref.tolist())
    return 0.0 if den == 0 and num == 0 else (math.inf if den == 0 else num / den)


def _distance_l2(cur, prev):
    diff, ref = G.l1_terms(cur, prev)
    num, den = math.sqrt(math.fsum((diff ** 2).tolist())), math.sqrt(math.fsum((ref ** 2).tolist()))
    return 0.0 if den == 0 and num == 0 else (math.inf if den == 0 else num / den)


def _update_with(strict=True, reset=True):
    def f(state, d, delta):
        acc = state.acc if d is None else state.acc + d
        low = acc < delta if strict else acc <= delta
        if low:
            return G.GbsState(acc, G.GBS_LOW_BITS, state.step + 1)
        return G.GbsState(0.0 if reset else acc, G.GBS_HIGH_BITS, state.step + 1)
    return f


@dataclass(frozen=True)
class _LowStart(G.GbsState):
    bits: int = G.GBS_LOW_BITS


MUTANTS = {
    "normalised_by_current_output": ("l1_distance", _distance_by_current),
    "l2_instead_of_l1": ("l1_distance", _distance_l2),
    "equality_stays_low": ("gbs_update", _update_with(strict=False)),
    "no_reset_on_switch": ("gbs_update", _update_with(reset=False)),
    "first_step_low": ("GbsState", _LowStart),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(G, attr, fn)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(G)
        except Exception as e:  # noqa: BLE001 - any failure of a pin counts
            caught.append((pin.__name__, type(e).__name__))
    assert caught, f"no pin catches the mutant {name}"
