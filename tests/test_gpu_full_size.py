"""Full-size parity on every seeded configuration: every element compared.

The bar of the rotated layer (DVD-Quant, "Resumen técnico" §2.B, the operation
whose result must match): packed codes, per-token and per-channel scales and
int32 accumulators bit-identical to the CPU oracle, bf16 outputs within one
bf16 ulp (and, since both sides take the epilogue's binary32 steps in the same
order, expected bit-identical).  Here that is checked on ALL rows and columns
of the HunyuanVideo-like QKV, the Wan-14B-like FFN (W4A4 with packed and with
byte-stored activation codes, W8A8, W4A8, W4A6) and the four layers of the Wan
block chain, in the launch configuration the benchmark times; and the same
for the two other weight/activation formats of the Wan FFN layer: weights on
bounded-init refined grids (asymmetric, DVD-Quant §2.A) and the SD4 block
format with the activation decomposition (SemanticDialect §2.A-§2.B).

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
from oracle import bgr_oracle as B
from oracle import qs_oracle as O
from oracle import sd4_oracle as S

import oracle_pool as P

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


def test_full_size_bgr_every_element():
    """The Wan FFN layer with its weights on bounded-init refined grids
    (DVD-Quant, "Resumen técnico" §2.A: asymmetric per-channel codes, the
    default 64 candidates and 8 refinement steps) and symmetric per-token
    activations with their code sums, as the benchmark times it: every weight
    code, scale and offset, every token's codes, scale and code sum, every
    int32 accumulator and every bf16 output against the oracle."""
    cfg = I.WAN_FFN
    d = I.make_layer(cfg)
    M, K, N, bits, alpha = cfg.M, cfg.K, cfg.N, cfg.bits, cfg.alpha
    J, T = B.BGR_DEFAULT_CANDIDATES, B.BGR_DEFAULT_ITERATIONS
    x, w, b = d["x"].cuda(), d["w"].cuda(), d["bias"].cuda()
    wp, ws, wo = qs.pack_weights_bgr(w, bits, J, T)
    xp, xs, xr = qs.quant_act_rowsum(x, bits, alpha)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    qs.qs_qlinear_asym(xp, xs, xr, wp, ws, wo, b, M, N, K, bits, out)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    qs.qs_qgemm_s32_asym(xp, xr, wp, wo, M, N, K, bits, acc)
    torch.cuda.synchronize()
    assert qs.qs_device_error() == 0
    del x, w, b

    s, sw, off = P.bgr_pack_weights(I.bf16_bits(d["w"]), bits, J, T)
    assert np.array_equal(ws.cpu().numpy().view(np.uint32), sw.view(np.uint32)), "w scales"
    assert np.array_equal(wo.cpu().numpy(), off), "w offsets"
    assert np.array_equal(wp.cpu().numpy(), O.pack(s, bits)), "w codes"
    bb = I.bf16_bits(d["bias"])
    xbits = I.bf16_bits(d["x"])
    for r0 in range(0, M, ROW_BLOCK):
        r1 = min(M, r0 + ROW_BLOCK)
        tag = f"rows {r0}:{r1}"
        qa, sa = O.quant_act(xbits[r0:r1], bits, alpha)
        assert np.array_equal(xs[r0:r1].cpu().numpy().view(np.uint32), sa.view(np.uint32)), \
            f"x scales, {tag}"
        assert np.array_equal(xp[r0:r1].cpu().numpy(), O.pack(qa, bits)), f"x codes, {tag}"
        assert np.array_equal(xr[r0:r1].cpu().numpy().astype(np.int64), B.code_rowsums(qa)), \
            f"code sums, {tag}"
        want_acc = B.asym_accumulators(qa, s, off, gemm=O.int_gemm_f64)
        ga = acc[r0:r1].cpu().numpy().astype(np.int64)
        if not np.array_equal(ga, want_acc):
            bad = np.argwhere(ga != want_acc)
            raise AssertionError(f"int32 accumulators differ at {len(bad)} places, "
                                 f"first {(bad[:4] + [r0, 0]).tolist()}, {tag}")
        want = O.epilogue(want_acc, sa, sw, bb)
        dd = np.abs(_ordered(_u16(out[r0:r1])) - _ordered(want))
        assert dd.max(initial=0) <= 1, f"bf16 outputs beyond 1 ulp, {tag}"
        assert (dd == 0).all(), f"{int((dd != 0).sum())} outputs differ by 1 ulp, {tag}"


def _e4m3_table():
    # the e4m3 byte of every (dialect, code): sign and L/8 of the oracle's
    # formatbook (exact in e4m3), encoded by torch's float8 conversion
    L = S.formatbook()
    mag = L.astype(np.float64) / 8.0
    val = np.concatenate([mag, -mag], axis=1)                 # code = sign << 3 | level
    return torch.from_numpy(val).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _sd4_bound_check(got_bits, y, bias_f64, S_abs, terms, tag):
    """|got - (y + bias)| <= terms 2^-23 S_abs + one bf16 ulp of got: binary32
    accumulation of exact products (at most `terms` roundings of 2^-24
    relative, doubled for the final additions), then the bf16 rounding."""
    got = O.bf16_bits_to_f32(got_bits).astype(np.float64)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(got), 2.0 ** -126))) - 7)
    excess = np.abs(got - (y + bias_f64)) - (terms * 2.0 ** -23 * S_abs + ulp)
    assert (excess <= 0).all(), f"outputs beyond the bound by up to {excess.max()}, {tag}"


def test_full_size_sd4_every_element():
    """The Wan FFN layer in the SD4 block format (SemanticDialect, "Resumen
    técnico" §2.A) in every form the benchmark times, and its activation
    decomposition of a seeded 1/16 of the tokens (§2.B): every activation and
    weight code and block word, every e4m3 byte and decoded bf16 weight
    bit-identical to the oracle; every output of the codes form (with the
    e4m3 forms, also with pre-arranged scale tiles, bit-identical to it) and of the bf16-weight form, and every
    decomposed row's codes, block words and outputs, within the
    binary32-accumulation bound of the oracle's exact-product layer, with
    more than 99 % of them bit-identical to the oracle's rounding."""
    cfg = I.WAN_FFN
    d = I.make_layer(cfg)
    M, K, N = cfg.M, cfg.K, cfg.N
    x, w, b = d["x"].cuda(), d["w"].cuda(), d["bias"].cuda()
    cx, mx = qs.sd4_quant(x)
    cw, mw = qs.sd4_quant(w)
    x8, mx8 = qs.sd4_quant_e4m3(x)
    w8 = qs.sd4_decode_e4m3(cw, mw)
    wdec = qs.sd4_decode(cw, mw)
    outs = {k: torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            for k in ("codes", "e4m3w", "e4m3", "wdec")}
    qs.qs_sd4_linear(cx, mx, cw, mw, b, M, N, K, outs["codes"])
    qs.qs_sd4_linear_e4m3w(cx, mx, w8, mw, b, M, N, K, outs["e4m3w"])
    qs.qs_sd4_linear_e4m3(x8, mx8, w8, mw, b, M, N, K, outs["e4m3"])
    qs.qs_sd4_linear_wdec(cx, mx, wdec, b, M, N, K, outs["wdec"])
    out_tiles = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    qs.qs_sd4_linear_e4m3_tiles(x8, qs.sd4_scale_tiles(mx8, False), w8,
                                qs.sd4_scale_tiles(mw, True), b, M, N, K, out_tiles)
    rows = I.salient_rows(M, cfg.seed)
    rt = torch.tensor(rows, dtype=torch.int32, device="cuda")
    codes2, meta2 = qs.sd4_quant_decomp(x, rt)
    outd = outs["e4m3"].clone()
    qs.qs_sd4_linear_decomp(codes2, meta2, rt, len(rows), None, mw, w8, b, M, N, K, outd)
    torch.cuda.synchronize()
    assert qs.qs_device_error() == 0
    assert torch.equal(mx8, mx), "block words of the e4m3 quantiser"
    ref16 = outs["codes"].view(torch.int16)
    assert torch.equal(outs["e4m3w"].view(torch.int16), ref16), "e4m3-weight form"
    assert torch.equal(outs["e4m3"].view(torch.int16), ref16), "e4m3 form"
    assert torch.equal(out_tiles.view(torch.int16), ref16), "e4m3 form with scale tiles"
    del out_tiles
    plain = torch.ones(M, dtype=torch.bool, device="cuda")
    plain[rt.long()] = False
    assert torch.equal(outd.view(torch.int16)[plain], ref16[plain]), \
        "the decomposition writes only the salient rows"
    x8_host = x8.cpu().numpy()
    del x, w, b, x8

    # weights: codes, block words, e4m3 bytes, bf16 decode
    table = _e4m3_table()
    xbits, wbits = I.bf16_bits(d["x"]), I.bf16_bits(d["w"])
    cwo, ewo, dwo = P.sd4_quantize_rows(wbits)
    assert np.array_equal(cw.cpu().numpy(), S.pack_codes(cwo)), "w codes"
    assert np.array_equal(mw.cpu().numpy().view(np.uint16), S.pack_meta(ewo, dwo)), "w words"
    assert np.array_equal(w8.cpu().numpy(), table[np.repeat(dwo, 32, axis=1), cwo]), "w e4m3"
    wh = S.dequantize(cwo, ewo, dwo)
    assert np.array_equal(_u16(wdec), O.f32_to_bf16_bits(wh.astype(np.float32))), "w decode"
    del cwo, ewo, dwo
    absw = np.abs(wh).T
    bb = I.bf16_bits(d["bias"])
    bias = O.bf16_bits_to_f32(bb).astype(np.float64)[None, :]

    # activations and the layer, by row blocks
    qx = P.sd4_quantize_rows(xbits)
    same = {"codes": 0, "wdec": 0}
    for r0 in range(0, M, ROW_BLOCK):
        r1 = min(M, r0 + ROW_BLOCK)
        tag = f"rows {r0}:{r1}"
        c, e, dia = (a[r0:r1] for a in qx)
        assert np.array_equal(cx[r0:r1].cpu().numpy(), S.pack_codes(c)), f"x codes, {tag}"
        assert np.array_equal(mx[r0:r1].cpu().numpy().view(np.uint16), S.pack_meta(e, dia)), \
            f"x words, {tag}"
        assert np.array_equal(x8_host[r0:r1], table[np.repeat(dia, 32, axis=1), c]), \
            f"x e4m3, {tag}"
        xh = S.dequantize(c, e, dia)
        y, want = S.layer_outputs(xh, wh, bb, exact=False)
        S_abs = np.abs(xh) @ absw
        for k in same:
            got = _u16(outs[k][r0:r1])
            _sd4_bound_check(got, y, bias, S_abs, K, f"{k} form, {tag}")
            same[k] += int((got == want).sum())
    for k, n in same.items():
        assert n > 0.99 * M * N, f"{k} form: only {n / (M * N):.4f} bit-identical to the oracle"

    # the decomposed rows
    dec = P.sd4_decompose_rows(xbits[rows])
    want_c, want_m = S.pack_decomp(dec)
    assert np.array_equal(codes2.cpu().numpy(), want_c), "decomposed codes"
    assert np.array_equal(meta2.cpu().numpy().view(np.uint16), want_m), "decomposed words"
    y, want = S.layer_outputs(dec["x_hat"] + dec["d_hat"], wh, bb, exact=False)
    S_abs = np.abs(dec["x_hat"]) @ absw + np.abs(dec["d_hat"]) @ absw
    got = _u16(outd[rt.long()])
    _sd4_bound_check(got, y, bias, S_abs, 2 * K, "decomposed rows")
    assert (got == want).mean() > 0.99, "decomposed rows bit-identical to the oracle"
