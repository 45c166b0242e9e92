"""How much the two readings of the quantiser's rounding step differ.

TEST INFRASTRUCTURE ONLY (part of the oracle): it imports the oracle and the
seeded input generator and nothing else of this repository.

DVD-Quant ("Resumen técnico" §2.B) says only that the scale factors are
computed at run time from the rotated activations; it fixes neither a
division by the scale nor a multiplication by its reciprocal.  Two plain
readings of q = round(u / s) exist:

  division    q = clamp(rint_half_even(fl(u / s)), -qmax, qmax),
              s = fl(t / qmax), t = fl(alpha * amax)  (one IEEE division per code)
  multiplier  q = clamp(rint_half_even(u * inv), -qmax, qmax), inv = fl(qmax / t),
              the exact product rounded once            (one division per row)

The oracle and the CUDA path take the multiplier reading.  This script
counts, on the seeded configurations, how many codes the two readings give
differently, so that the choice can be seen to be immaterial:

    python -m oracle.quantiser_readings [--rows R]

(R limits the token rows per configuration; default all rows.)
"""

from __future__ import annotations

import argparse
import sys

import numpy as np

from oracle import qs_oracle as O


def codes_division(u: np.ndarray, bits: int, alpha: float) -> np.ndarray:
    """The division reading: fl(u / s) in binary32, then round half to even."""
    qmax = np.float32(O.QMAX[bits])
    amax = np.max(np.abs(u), axis=1).astype(np.float32)
    t = (np.float32(alpha) * amax).astype(np.float32)
    zero = t < O.ZERO_ROW_T
    s = np.where(zero, np.float32(1), t / qmax).astype(np.float32)
    r = (u / s[:, None]).astype(np.float32)
    q = np.clip(np.rint(r), -qmax, qmax)
    q[zero] = 0
    return q.astype(np.int8)


def codes_multiplier(u: np.ndarray, bits: int, alpha: float) -> np.ndarray:
    """The oracle's own reading (its row scales and quantiser)."""
    _, inv = O.row_scales(u, bits, alpha)
    return O.quantize_with_scale(u, inv, bits)


def compare(x_bits: np.ndarray, bits: int, alpha: float, block: int = 4096) -> dict:
    rows = x_bits.shape[0]
    diff = rows_hit = total = 0
    max_step = 0
    for r0 in range(0, rows, block):
        u = O.fwht128_blocks(O.bf16_bits_to_f32(x_bits[r0:r0 + block]))
        a = codes_division(u, bits, alpha)
        b = codes_multiplier(u, bits, alpha)
        d = a != b
        diff += int(d.sum())
        rows_hit += int(d.any(axis=1).sum())
        total += d.size
        if d.any():
            max_step = max(max_step, int(np.abs(a.astype(np.int16) - b.astype(np.int16)).max()))
    return {"codes": total, "differ": diff, "rows": rows, "rows_with_a_difference": rows_hit,
            "max_code_step": max_step}


def _gelu_table() -> np.ndarray:
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = (pats & 0x7F80) != 0x7F80
    table = np.zeros(65536, np.uint16)
    table[finite] = O.gelu_erf_bf16(pats[finite])
    return table


def main(argv=None) -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--rows", type=int, default=None)
    a = ap.parse_args(argv)
    import os
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from bit_quantized_linear_hadamard_b200 import inputs as I

    cases = []
    for cfg in (I.TINY, I.HY_QKV, I.WAN_FFN, I.WAN_FFN_W8, *I.MIXED_CONFIGS):
        d = I.make_layer(cfg, M=min(cfg.M, a.rows) if a.rows else None)
        cases.append((cfg.name + " (activations)", I.bf16_bits(d["x"]), cfg.act_bits, cfg.alpha))
        cases.append((cfg.name + " (weights)", I.bf16_bits(d["w"]), cfg.bits, 1.0))
    ch = I.make_chain(I.WAN_CHAIN, M=min(I.WAN_CHAIN.M, a.rows) if a.rows else None)
    up = None
    for L in ch["layers"]:
        if L["x"] is not None:
            xb = I.bf16_bits(L["x"])
        else:
            # down's input: GELU of the oracle's own up-projection output
            xb = _gelu_table()[up]
        cases.append((f"{I.WAN_CHAIN.name} {L['name']} (activations)", xb, L["bits"], ch["alpha"]))
        cases.append((f"{I.WAN_CHAIN.name} {L['name']} (weights)", I.bf16_bits(L["w"]),
                      L["bits"], 1.0))
        if L["name"] == "ffn_up":
            qw, sw = O.pack_weights(I.bf16_bits(L["w"]), L["bits"])
            bb = I.bf16_bits(L["bias"])
            outs = []
            for r0 in range(0, xb.shape[0], 4096):
                qa, sa = O.quant_act(xb[r0:r0 + 4096], L["bits"], ch["alpha"])
                outs.append(O.epilogue(O.int_gemm_f64(qa, qw), sa, sw, bb))
            up = np.concatenate(outs)
    for name, xb, bits, alpha in cases:
        r = compare(xb, bits, alpha)
        print(f"{name}: {bits}-bit, alpha {alpha}: {r['differ']} of {r['codes']} codes differ "
              f"({r['rows_with_a_difference']} of {r['rows']} rows), "
              f"largest difference {r['max_code_step']}", flush=True)


if __name__ == "__main__":
    main()
