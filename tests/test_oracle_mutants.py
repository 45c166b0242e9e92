"""Plant plausible mistakes in the oracle (on the CPU) and require a pin to catch each.

Each mutant replaces one oracle function for the duration of the test; the pin
suite of ``test_oracle_pins.py`` is then run against the mutated oracle and at
least one pin must fail.
"""

import numpy as np
import pytest

from oracle import qs_oracle as O
import test_oracle_pins as P


def _fwht_with(stage_fn, stages=(1, 2, 4, 8, 16, 32, 64)):
    def f(x):
        x = np.ascontiguousarray(x, dtype=np.float32)
        R, K = x.shape
        v = x.reshape(R, K // 128, 128).copy()
        for h in stages:
            w = v.reshape(R, K // 128, 128 // (2 * h), 2, h)
            a = w[:, :, :, 0, :].copy()
            b = w[:, :, :, 1, :].copy()
            lo, hi = stage_fn(a, b)
            w[:, :, :, 0, :] = lo
            w[:, :, :, 1, :] = hi
        return v.reshape(R, K)
    return f


def _quantize_with(round_fn=np.rint, lo_extra=0):
    def f(u, inv, bits):
        qmax = np.float32(O.QMAX[bits])
        r = u.astype(np.float64) * np.asarray(inv, dtype=np.float32).astype(np.float64)[:, None]
        q = round_fn(r)
        q = np.minimum(np.maximum(q, -qmax - lo_extra), qmax)
        return q.astype(np.int8)
    return f


def _scales_with(alpha_used=True, div=None):
    def f(u, bits, alpha):
        amax = np.max(np.abs(u), axis=1).astype(np.float32)
        t = ((np.float32(alpha) if alpha_used else np.float32(1)) * amax).astype(np.float32)
        d = np.float32(O.QMAX[bits] if div is None else div(bits))
        zero = t == 0
        safe = np.where(zero, np.float32(1), t)
        return (np.where(zero, 0, t / d).astype(np.float32),
                np.where(zero, 0, d / safe).astype(np.float32))
    return f


def _per_block_quantize_rows(x_bits, bits, alpha, rotate=True):
    x = O.bf16_bits_to_f32(np.asarray(x_bits))
    u = O.fwht128_blocks(x) if rotate else x.copy()
    R, K = u.shape
    ub = u.reshape(R * (K // 128), 128)
    s, inv = O.row_scales(ub, bits, alpha)
    q = O.quantize_with_scale(ub, inv, bits).reshape(R, K)
    return q, s.reshape(R, K // 128)[:, 0].copy()


def _pack_swapped(q, bits):
    if bits == 8:
        return np.asarray(q, dtype=np.int8).view(np.uint8).copy()
    nib = np.asarray(q, dtype=np.int8).astype(np.uint8) & np.uint8(0x0F)
    return (nib[:, 1::2] | (nib[:, 0::2] << np.uint8(4))).astype(np.uint8)


def _unpack_no_sign(p, bits):
    p = np.asarray(p, dtype=np.uint8)
    if bits == 8:
        return p.view(np.int8).copy()
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.int8)
    out[:, 0::2] = (p & np.uint8(0x0F)).astype(np.int8)
    out[:, 1::2] = (p >> np.uint8(4)).astype(np.int8)
    return out


def _epilogue_with(fold_bias_first=False, drop_bias=False):
    def f(acc, s_a, s_w, bias_bits):
        s_a = np.asarray(s_a, dtype=np.float32)
        s_w = np.asarray(s_w, dtype=np.float32)
        accf = np.asarray(acc, dtype=np.int64).astype(np.float32)
        b = np.zeros(s_w.shape, np.float32) if (bias_bits is None or drop_bias) else O.bf16_bits_to_f32(bias_bits)
        if fold_bias_first:
            y = (s_a[:, None] * s_w[None, :]) * (accf + b[None, :])
        else:
            y = (s_a[:, None] * s_w[None, :]) * accf + b[None, :]
        return O.f32_to_bf16_bits(y)
    return f


def _bf16_truncate(x):
    f = np.ascontiguousarray(x, dtype=np.float32)
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def _pack_weights_no_fold(w_bits, bits, rotate=True):
    return O.quantize_rows(w_bits, bits, 1.0, rotate)


def _quantize_double_rounding(u, inv, bits):
    qmax = np.float32(O.QMAX[bits])
    r = (np.asarray(u, np.float32) * np.asarray(inv, np.float32)[:, None]).astype(np.float32)
    return np.minimum(np.maximum(np.rint(r), -qmax), qmax).astype(np.int8)


def _pack_six_as_nibbles(q, bits):
    return _REAL_PACK(q, 4 if bits == 6 else bits)


_REAL_PACK = O.pack

MUTANTS = {
    "product_rounded_to_binary32_first": ("quantize_with_scale", _quantize_double_rounding),
    "fwht_sign_flipped": ("fwht128_blocks", _fwht_with(lambda a, b: (a + b, b - a))),
    "fwht_stage_dropped": ("fwht128_blocks", _fwht_with(lambda a, b: (a + b, a - b), (1, 2, 4, 8, 16, 32))),
    "fwht_halves_swapped": ("fwht128_blocks", _fwht_with(lambda a, b: (a - b, a + b))),
    "scale_ignores_alpha": ("row_scales", _scales_with(alpha_used=False)),
    "scale_divides_by_2^(b-1)": ("row_scales", _scales_with(div=lambda b: 2 ** (b - 1))),
    "round_half_away": ("quantize_with_scale", _quantize_with(lambda r: np.sign(r) * np.floor(np.abs(r) + 0.5))),
    "truncate_not_round": ("quantize_with_scale", _quantize_with(np.trunc)),
    "asymmetric_clamp": ("quantize_with_scale", _quantize_with(lo_extra=1)),
    "per_block_scale": ("quantize_rows", _per_block_quantize_rows),
    "nibbles_swapped": ("pack", _pack_swapped),
    "unpack_without_sign": ("unpack", _unpack_no_sign),
    "gemm_one_operand_k_reversed": ("int_gemm", lambda a, w: np.asarray(a, np.int64) @ np.asarray(w, np.int64)[:, ::-1].T),
    "bias_inside_scale": ("epilogue", _epilogue_with(fold_bias_first=True)),
    "bias_dropped": ("epilogue", _epilogue_with(drop_bias=True)),
    "bf16_truncation": ("f32_to_bf16_bits", _bf16_truncate),
    "weight_scale_not_folded": ("pack_weights", _pack_weights_no_fold),
    "six_bit_qmax_is_2^5": ("QMAX", {4: 7, 6: 32, 8: 127}),
    "six_bit_codes_as_nibbles": ("pack", _pack_six_as_nibbles),
    "blas_gemm_in_binary32": ("int_gemm_f64", lambda a, w: (np.asarray(a, np.float32) @ np.asarray(w, np.float32).T).astype(np.int64)),
    "blas_gemm_operand_transposed": ("int_gemm_f64", lambda a, w: (np.asarray(a, np.float64) @ np.asarray(w, np.float64)[:, ::-1].T).astype(np.int64)),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    caught = []
    for pin in P.ALL_PINS:
        try:
            pin(O)
        except Exception as e:  # noqa: BLE001 - any failure of a pin counts
            caught.append((pin.__name__, type(e).__name__))
    assert caught, f"no pin catches the mutant {name}"
