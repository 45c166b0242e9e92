"""Full-size parity on every seeded configuration: every element compared.

The bar of the rotated layer (DVD-Quant, "Resumen técnico" §2.B, the operation
whose result must match): packed codes, per-token and per-channel scales and
int32 accumulators bit-identical to the CPU oracle, bf16 outputs within one
bf16 ulp (and, since both sides take the epilogue's binary32 steps in the same
order, expected bit-identical).  Here that is checked on ALL rows and columns
of the HunyuanVideo-like QKV, the Wan-14B-like FFN (W4A4 with packed and with
byte-stored activation codes, W8A8, W4A8, W4A6) and the four layers of the Wan
block chain, in the launch configuration the benchmark times.

The oracle runs block by block over the token rows (its quantiser, its
binary64-BLAS accumulators -- exact, see ``int_gemm_f64`` -- and its
epilogue), and each block is compared with the same rows of the device
results.  Nothing here comes from the CUDA path except the values compared.
"""

import numpy as np
import pytest
import torch

import bit_quantized_linear_hadamard_b200 as qs
from bit_quantized_linear_hadamard_b200 import build as qs_build
from bit_quantized_linear_hadamard_b200 import inputs as I
from oracle import qs_oracle as O

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

ROW_BLOCK = 4096


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    qs_build.build()
    qs.load()
    yield
    assert qs.qs_device_error() == 0, "a kernel reported a bounded-wait timeout"


def _u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _ordered(b):
    b = np.asarray(b, dtype=np.int32)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def full_parity(x, w, bias, bits_w, alpha, bits_x, layouts=(0,)):
    """Runs the layer on the device for each activation-code layout (x_flags)
    and compares every code, scale, accumulator and output with the oracle.

    Returns the device output of the first layout (bf16, on the device) and
    the count of outputs compared.
    """
    K = x.shape[1]
    N = w.shape[0]
    M = x.shape[0]
    xd, wd, bd = x.cuda(), w.cuda(), bias.cuda()
    wp, ws = qs.pack_weights(wd, bits_w)
    runs = []
    for flags in layouts:
        sx = qs.storage_bits(bits_x, flags)
        xp, xs = qs.quant_act(xd, bits_x, alpha, flags)
        out = qs.qlinear(xp, xs, wp, ws, bd, sx, K, bits_w=bits_w)
        acc = qs.qgemm_s32(xp, wp, sx, K, bits_w=bits_w)
        runs.append({"flags": flags, "sx": sx, "xp": xp, "xs": xs, "out": out, "acc": acc})
    torch.cuda.synchronize()
    assert qs.qs_device_error() == 0

    # weights: every code and channel scale
    qw, sw = O.pack_weights(I.bf16_bits(w), bits_w)
    assert np.array_equal(ws.cpu().numpy().view(np.uint32), sw.view(np.uint32)), "w scales"
    assert np.array_equal(wp.cpu().numpy(), O.pack(qw, bits_w)), "w codes"
    bb = I.bf16_bits(bias)
    xbits = I.bf16_bits(x)

    for r0 in range(0, M, ROW_BLOCK):
        r1 = min(M, r0 + ROW_BLOCK)
        qa, sa = O.quant_act(xbits[r0:r1], bits_x, alpha)
        acc = O.int_gemm_f64(qa, qw)
        want = O.epilogue(acc, sa, sw, bb)
        for g in runs:
            tag = f"rows {r0}:{r1}, layout {g['flags']}"
            gs = g["xs"][r0:r1].cpu().numpy()
            assert np.array_equal(gs.view(np.uint32), sa.view(np.uint32)), f"x scales, {tag}"
            gp = g["xp"][r0:r1].cpu().numpy()
            assert np.array_equal(gp, O.pack(qa, g["sx"])), \
                f"x codes, {tag}"
            ga = g["acc"][r0:r1].cpu().numpy()
            if not np.array_equal(ga.astype(np.int64), acc):
                bad = np.argwhere(ga.astype(np.int64) != acc)
                raise AssertionError(f"int32 accumulators differ at {len(bad)} places, "
                                     f"first {(bad[:4] + [r0, 0]).tolist()}, {tag}")
            got = _u16(g["out"][r0:r1])
            d = np.abs(_ordered(got) - _ordered(want))
            assert d.max(initial=0) <= 1, f"bf16 outputs beyond 1 ulp, {tag}"
            assert (d == 0).all(), f"{int((d != 0).sum())} outputs differ by 1 ulp, {tag}"
    return runs[0]["out"], M * N


CONFIGS = [I.HY_QKV, I.WAN_FFN_W8, *I.MIXED_CONFIGS]


@pytest.mark.parametrize("cfg", CONFIGS, ids=lambda c: c.name)
def test_full_size_config_every_element(cfg):
    d = I.make_layer(cfg)
    _, n = full_parity(d["x"], d["w"], d["bias"], cfg.bits, cfg.alpha, cfg.act_bits)
    assert n == cfg.M * cfg.N


def test_full_size_wan_ffn_w4a4_both_layouts_every_element():
    """The Wan FFN W4A4 layer with packed activation codes (two per byte, the
    4x4 GEMM) and with byte-stored codes (the mixed-storage GEMM), both
    against one oracle pass."""
    cfg = I.WAN_FFN
    d = I.make_layer(cfg)
    full_parity(d["x"], d["w"], d["bias"], cfg.bits, cfg.alpha, cfg.bits,
                layouts=(0, qs.QS_FLAG_BYTE_CODES))


def _gelu_table():
    # the oracle's GELU of every bf16 pattern; the chain's down-projection
    # input is compared through this table (the oracle evaluated per pattern)
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = (pats & 0x7F80) != 0x7F80
    table = np.zeros(65536, np.uint16)
    table[finite] = O.gelu_erf_bf16(pats[finite])
    return table, finite


def test_full_size_block_chain_every_element():
    ch = I.make_chain(I.WAN_CHAIN)
    alpha = ch["alpha"]
    up_out = None
    table, finite = _gelu_table()
    for i, L in enumerate(ch["layers"]):
        if i < 3:
            x = L["x"]
        else:
            xg = qs.gelu(up_out)
            torch.cuda.synchronize()
            ub = _u16(up_out)
            gb = _u16(xg)
            assert finite[ub].all(), "the up-projection output is finite"
            d = np.abs(_ordered(gb) - _ordered(table[ub]))
            assert d.max() <= 1, "GELU within 1 bf16 ulp of the oracle on every element"
            x = xg.cpu()
            del xg
        out, _ = full_parity(x, L["w"], L["bias"], L["bits"], alpha, L["bits"])
        if L["name"] == "ffn_up":
            up_out = out
        else:
            del out
        torch.cuda.empty_cache()
