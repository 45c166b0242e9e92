"""CPU oracle of δ-guided bit switching (δ-GBS) for the quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only the test-suite, the smoke check and the CPU-baseline
leg of the benchmark use it.  It shares no code with the CUDA library.

What the pages fix (DVD-Quant, "Resumen técnico" §2.C, "Cambio de Bits Guiado
por δ"; the lay summary's "Semáforo de Precisión" says the same): the bit width
of the layer is chosen per denoising step from how much its output features
change.  The normalised L1 distance between consecutive output features is
monitored and accumulated; while the accumulated change stays below a
threshold δ the layer runs at low precision (4 bits); once it exceeds δ the
layer switches to high precision (8 bits) and the accumulator is reset.

Readings taken where the pages are silent:

* Distance: d_t = sum_i |y_t[i] - y_{t-1}[i]| / sum_i |y_{t-1}[i]| over every
  element of the layer's bf16 output (normalised by the previous output).  Each
  term is the binary64 difference of the two bf16 values (bf16 -> binary64 is
  exact); both sums are the exact sums rounded once to binary64 (math.fsum),
  then one binary64 division.  A zero denominator gives d = 0 if the numerator
  is 0 too, else +inf.
* Accumulator and decision, taken after every step t: acc = acc + d_t
  (binary64; the first step has no previous output and adds nothing); the
  next step runs at 4 bits if acc < δ, otherwise at 8 bits with acc reset
  to 0.  "Below δ → low precision" is read as strict, so acc == δ switches.
* The first step (t = 0) runs at 8 bits: there is no change to measure yet and
  the high-precision mode is the safe one.
* One accumulator per layer; the decision for step t+1 uses the outputs of
  steps t and t-1 of the same layer.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

from .qs_oracle import bf16_bits_to_f32, qlinear

GBS_LOW_BITS = 4
GBS_HIGH_BITS = 8


def l1_terms(cur_bits: np.ndarray, prev_bits: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """|cur - prev| and |prev| per element, in binary64, from bf16 bit patterns."""
    a = bf16_bits_to_f32(np.asarray(cur_bits)).astype(np.float64).ravel()
    b = bf16_bits_to_f32(np.asarray(prev_bits)).astype(np.float64).ravel()
    return np.abs(a - b), np.abs(b)


def l1_distance(cur_bits: np.ndarray, prev_bits: np.ndarray) -> float:
    """Normalised L1 distance between consecutive outputs (see the module header)."""
    diff, ref = l1_terms(cur_bits, prev_bits)
    num = math.fsum(diff.tolist())
    den = math.fsum(ref.tolist())
    if den == 0.0:
        return 0.0 if num == 0.0 else math.inf
    return num / den


@dataclass(frozen=True)
class GbsState:
    acc: float = 0.0          # accumulated change since the last switch to 8 bits
    bits: int = GBS_HIGH_BITS  # width of the next step
    step: int = 0             # steps completed


def gbs_update(state: GbsState, d: float | None, delta: float) -> GbsState:
    """The decision after one step: add its distance (None for the first step,
    which has no previous output) and choose the next step's width."""
    acc = state.acc if d is None else state.acc + d
    if acc < delta:
        return GbsState(acc, GBS_LOW_BITS, state.step + 1)
    return GbsState(0.0, GBS_HIGH_BITS, state.step + 1)


def gbs_schedule(distances, delta: float) -> list[int]:
    """Widths of steps 0..len(distances) for the distances d_1, d_2, ... measured
    after steps 1, 2, ... (the decision after step 0 has no distance)."""
    s = GbsState()
    bits = [s.bits]
    s = gbs_update(s, None, delta)
    bits.append(s.bits)
    for d in distances:
        s = gbs_update(s, d, delta)
        bits.append(s.bits)
    return bits


def gbs_run(xs_bits, w_bits, bias_bits, alpha: float, delta: float):
    """One layer over consecutive steps with δ-GBS: step t quantises its input
    at the width chosen after step t-1 (weights prepared at both widths).
    Returns the widths used, the bf16 outputs, the distances and the states."""
    state = GbsState()
    used, outs, dists, states = [], [], [], []
    prev = None
    for x in xs_bits:
        used.append(state.bits)
        y = qlinear(x, w_bits, bias_bits, state.bits, alpha)["out"]
        d = None if prev is None else l1_distance(y, prev)
        state = gbs_update(state, d, delta)
        outs.append(y)
        dists.append(d)
        states.append(state)
        prev = y
    return {"bits": used, "out": outs, "d": dists, "states": states}
