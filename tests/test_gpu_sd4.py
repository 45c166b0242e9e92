"""GPU parity of the SD4 block format (SemanticDialect "Resumen técnico" §2.A)
through the C ABI, against the oracle (this library's formatbook; parity
against the pages is unpinned: they print no dialect values).

Bar: codes and block words (exponent, dialect) bit-identical."""

import numpy as np
import pytest
import torch

import bit_quantized_linear_hadamard_b200 as qs
from bit_quantized_linear_hadamard_b200 import build as qs_build
from bit_quantized_linear_hadamard_b200 import inputs as I
from oracle import qs_oracle as O
from oracle import sd4_oracle as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    qs_build.build()
    qs.load()
    yield
    assert qs.qs_device_error() == 0, "a kernel reported a bounded-wait timeout"


def check_quant(x):
    codes, meta = qs.sd4_quant(x.cuda())
    torch.cuda.synchronize()
    c, e, d = S.quantize_rows(I.bf16_bits(x))
    got_meta = meta.cpu().numpy().view(np.uint16)
    want_meta = S.pack_meta(e, d)
    if not np.array_equal(got_meta, want_meta):
        bad = np.argwhere(got_meta != want_meta)
        raise AssertionError(f"block words differ at {len(bad)}, first {bad[:5].tolist()}")
    assert np.array_equal(codes.cpu().numpy(), S.pack_codes(c)), "codes differ"


@pytest.mark.parametrize("M,K", [(1, 256), (7, 512), (33, 5120), (5, 13824), (3, 16384)])
def test_sd4_quant_bit_exact(M, K):
    d = I.make_shape(seed=M + K, M=M, K=K, N=16, bits=4, outlier_factor=30.0)
    check_quant(d["x"])
    check_quant(d["w"][:M] if d["w"].shape[0] >= M else d["w"])


def test_sd4_quant_edge_blocks():
    x = torch.randn(6, 512, generator=torch.Generator().manual_seed(3))
    x[0] = 0.0                                  # zero blocks
    x[1] = -0.0                                 # negative zeros
    x[2] = x[2] * 1e-39                         # subnormal blocks (exponent floor)
    x[3, :32] = torch.tensor([15 / 8 * 4.0] * 32)   # one level repeated
    x[4] = x[4] * 1e30                          # large exponents
    x[5, ::2] = 0.0
    check_quant(x.to(torch.bfloat16))


def _layer(M, N, K, seed, bias=True):
    d = I.make_shape(seed=seed, M=M, K=K, N=N, bits=4, outlier_factor=30.0)
    x, w = d["x"].cuda(), d["w"].cuda()
    b = d["bias"].cuda() if bias else None
    cx, mx = qs.sd4_quant(x)
    cw, mw = qs.sd4_quant(w)
    out = qs.sd4_linear(cx, mx, cw, mw, b, K)
    torch.cuda.synchronize()
    return d, (cx, mx, cw, mw), out


def _check_layer(d, dev, out, K, bias=True, exact=False):
    r = S.linear_sd4(I.bf16_bits(d["x"]), I.bf16_bits(d["w"]),
                     I.bf16_bits(d["bias"]) if bias else None, exact=exact)
    cx, mx, cw, mw = dev
    assert np.array_equal(cx.cpu().numpy(), S.pack_codes(r["codes_x"]))
    assert np.array_equal(mw.cpu().numpy().view(np.uint16), S.pack_meta(r["exp_w"], r["dia_w"]))
    got_bits = out.view(torch.int16).cpu().numpy().view(np.uint16)
    got = O.bf16_bits_to_f32(got_bits).astype(np.float64)
    b = O.bf16_bits_to_f32(I.bf16_bits(d["bias"])).astype(np.float64) if bias else 0.0
    exact_y = r["y"] + b
    # binary32 accumulation of exact products: at most K * 2^-23 of sum |products|,
    # plus the final bf16 rounding (one ulp of the result)
    S_abs = np.abs(r["x_hat"]) @ np.abs(r["w_hat"]).T
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(got), 2.0 ** -126))) - 7)
    allowed = K * 2.0 ** -23 * S_abs + ulp
    err = np.abs(got - exact_y)
    assert (err <= allowed).all(), f"max excess {np.max(err - allowed)}"
    same = float((got_bits == r["out"]).mean())
    assert same > 0.99, f"only {same:.4f} of outputs bit-identical to the oracle"
    return same


@pytest.mark.parametrize("M,N,K", [(1, 16, 256), (127, 272, 256), (256, 512, 512),
                                   (300, 768, 768), (513, 528, 1280)])
def test_sd4_linear_matches_oracle(M, N, K):
    d, dev, out = _layer(M, N, K, seed=M + N + K)
    _check_layer(d, dev, out, K)


def test_sd4_linear_exact_small_and_no_bias():
    d, dev, out = _layer(3, 16, 256, seed=5, bias=False)
    _check_layer(d, dev, out, 256, bias=False, exact=True)


def test_sd4_linear_extreme_exponents():
    # activation blocks with exponents down to -123 (the lowest exponent the
    # pair-table decode scales exactly) and up to +100; weights ordinary, so
    # every product stays a normal binary32 number
    g = torch.Generator().manual_seed(17)
    M, N, K = 64, 272, 512
    x = torch.randn(M, K, generator=g)
    scales = torch.tensor([2.0 ** -122, 2.0 ** -115, 2.0 ** -60, 1.0, 2.0 ** 40, 2.0 ** 100])
    x = x * scales[torch.arange(M) % len(scales)][:, None]
    w = torch.randn(N, K, generator=g) * 0.5
    d = {"x": x.to(torch.bfloat16), "w": w.to(torch.bfloat16),
         "bias": torch.zeros(N, dtype=torch.bfloat16)}
    cx, mx = qs.sd4_quant(d["x"].cuda())
    cw, mw = qs.sd4_quant(d["w"].cuda())
    out = qs.sd4_linear(cx, mx, cw, mw, None, K)
    torch.cuda.synchronize()
    e = (mx.cpu().numpy().view(np.uint16) & 0xFF).astype(np.int8)
    assert e.min() >= -123 and e.min() <= -120 and e.max() >= 100
    _check_layer(d, (cx, mx, cw, mw), out, K, bias=False)


@pytest.mark.parametrize("R,K", [(5, 256), (129, 5120)])
def test_sd4_decode_exact(R, K):
    d = I.make_shape(seed=R + K, M=R, K=K, N=16, bits=4, outlier_factor=30.0)
    codes, meta = qs.sd4_quant(d["x"].cuda())
    dec = qs.sd4_decode(codes, meta)
    torch.cuda.synchronize()
    c, e, dd = S.quantize_rows(I.bf16_bits(d["x"]))
    want = O.f32_to_bf16_bits(S.dequantize(c, e, dd).astype(np.float32))
    assert np.array_equal(dec.view(torch.int16).cpu().numpy().view(np.uint16), want)


@pytest.mark.parametrize("M,N,K", [(127, 272, 256), (300, 768, 768), (513, 528, 1280)])
def test_sd4_linear_e4m3_weights_identical_and_bf16_weights_within_bound(M, N, K):
    d, dev, out = _layer(M, N, K, seed=3 * M + N)
    cx, mx, cw, mw = dev
    # e4m3 weights: the same kernel arithmetic as the codes form
    w8 = qs.sd4_decode_e4m3(cw, mw)
    out8 = torch.empty_like(out)
    qs.qs_sd4_linear_e4m3w(cx, mx, w8, mw, d["bias"].cuda(), M, N, K, out8)
    # bf16 weights: the bf16 tensor-core kernel, its own accumulation order
    wdec = qs.sd4_decode(cw, mw)
    out16 = torch.empty_like(out)
    qs.qs_sd4_linear_wdec(cx, mx, wdec, d["bias"].cuda(), M, N, K, out16)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out8.view(torch.int16))
    _check_layer(d, dev, out16, K)


def _e4m3_of_codes(c, dd):
    L = S.formatbook()
    mag = L[np.repeat(dd, 32, axis=1), c & 7] / 8.0          # L/8, exact in e4m3
    val = np.where(c & 8, -mag, mag)
    return torch.from_numpy(val).to(torch.float8_e4m3fn).view(torch.uint8), val


@pytest.mark.parametrize("M,K", [(7, 256), (33, 5120), (5, 13824)])
def test_sd4_quant_e4m3_bit_exact(M, K):
    d = I.make_shape(seed=M + 3 * K, M=M, K=K, N=16, bits=4, outlier_factor=30.0)
    x8, meta = qs.sd4_quant_e4m3(d["x"].cuda())
    torch.cuda.synchronize()
    c, e, dd = S.quantize_rows(I.bf16_bits(d["x"]))
    assert np.array_equal(meta.cpu().numpy().view(np.uint16), S.pack_meta(e, dd))
    want, _ = _e4m3_of_codes(c, dd)
    assert torch.equal(x8.cpu(), want)


@pytest.mark.parametrize("M,N,K", [(127, 272, 256), (300, 768, 768), (513, 528, 1280),
                                   (1, 16, 256)])
def test_sd4_linear_e4m3_operands_identical(M, N, K):
    d, dev, out = _layer(M, N, K, seed=5 * M + N)
    cx, mx, cw, mw = dev
    x8, mx8 = qs.sd4_quant_e4m3(d["x"].cuda())
    w8 = qs.sd4_decode_e4m3(cw, mw)
    out8 = torch.empty_like(out)
    qs.qs_sd4_linear_e4m3(x8, mx8, w8, mw, d["bias"].cuda(), M, N, K, out8)
    torch.cuda.synchronize()
    assert torch.equal(mx8, mx)
    assert torch.equal(out.view(torch.int16), out8.view(torch.int16))
    _check_layer(d, dev, out8, K)


@pytest.mark.parametrize("R,K", [(5, 256), (129, 5120)])
def test_sd4_decode_e4m3_exact(R, K):
    d = I.make_shape(seed=R + 2 * K, M=R, K=K, N=16, bits=4, outlier_factor=30.0)
    codes, meta = qs.sd4_quant(d["x"].cuda())
    got = qs.sd4_decode_e4m3(codes, meta).cpu()
    torch.cuda.synchronize()
    c, e, dd = S.quantize_rows(I.bf16_bits(d["x"]))
    L = S.formatbook()
    mag = L[np.repeat(dd, 32, axis=1), c & 7] / 8.0          # L/8, exact in e4m3
    val = np.where(c & 8, -mag, mag)
    want = torch.from_numpy(val).to(torch.float8_e4m3fn).view(torch.uint8)
    # torch encodes -0.0 with the sign bit, as the kernel does for a negative level-0 code
    assert torch.equal(got, want)
    assert np.array_equal(got.view(torch.float8_e4m3fn).double().numpy(), val)


# ------------------------------------------------- activation decomposition (§2.B)

def _rows_tensor(rows):
    return torch.tensor(rows, dtype=torch.int32, device="cuda")


def check_decomp(x, rows):
    codes2, meta2 = qs.sd4_quant_decomp(x.cuda(), _rows_tensor(rows))
    torch.cuda.synchronize()
    dec = S.decompose_rows(I.bf16_bits(x), rows)
    want_c, want_m = S.pack_decomp(dec)
    got_m = meta2.cpu().numpy().view(np.uint16)
    if not np.array_equal(got_m, want_m):
        bad = np.argwhere(got_m != want_m)
        raise AssertionError(f"block words differ at {len(bad)}, first {bad[:5].tolist()}")
    assert np.array_equal(codes2.cpu().numpy(), want_c), "codes differ"
    return codes2, meta2, dec


@pytest.mark.parametrize("M,K,S_", [(7, 256, 7), (33, 5120, 12), (40, 13824, 9), (3, 32768, 2)])
def test_sd4_quant_decomp_bit_exact(M, K, S_):
    d = I.make_shape(seed=M + K + 1, M=M, K=K, N=16, bits=4, outlier_factor=30.0)
    rng = np.random.default_rng(M + K)
    rows = [0, M - 1] + rng.integers(0, M, S_ - 2).tolist() if S_ > 2 else [M - 1, 0][:S_]
    check_decomp(d["x"], rows)


def test_sd4_quant_decomp_edge_rows():
    g = torch.Generator().manual_seed(8)
    x = torch.randn(6, 512, generator=g)
    x[0] = 0.0                              # zero residual, zero blocks
    x[1] = -0.0
    x[2] = x[2] * 2.0 ** -118               # residuals at the exponent floor (subnormal binary32)
    x[3] = x[3] * 1e30
    x[2, 5] = 2.0 ** -130                   # rounds to level 0: a subnormal residual
    x[2, 40] = -3 * 2.0 ** -131
    x[4, ::3] = 0.0
    k = torch.arange(32, dtype=torch.float32)
    x[5, 64:96] = k * 2.0 ** -133 * (1 - 2 * (k % 2))   # a block of bf16 subnormals: e = -126
    x = x.to(torch.bfloat16)
    _, _, dec = check_decomp(x, [0, 1, 2, 3, 4, 5, 2])
    assert dec["delta"][2, 5] == 2.0 ** -130 and dec["exp_x"][5, 2] == -126


def test_sd4_decomp_reconstructs_two_scale_rows_exactly():
    # blocks x = a + b (levels at two scales, built as in the oracle's pins):
    # the device codes decode to x_hat + delta_hat = x exactly
    rng = np.random.default_rng(2)
    L = S.formatbook()
    R, K = 4, 512
    x = np.zeros((R, K))
    for r in range(R):
        for j in range(K // 32):
            e = int(rng.integers(-30, 30))
            nz = rng.choice(32, 20, replace=False)
            idx = rng.integers(0, 8, 20)
            idx[0] = 7
            x[r, 32 * j + nz] = (rng.choice([-1.0, 1.0], 20) * 15 / 8 * 2.0 ** e
                                 + rng.choice([-1.0, 1.0], 20) * L[21, idx] / 8 * 2.0 ** (e - 4))
    xt = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(xt.float().numpy().astype(np.float64), x)
    codes2, meta2, _ = check_decomp(xt, [3, 1, 0, 2])
    dec = qs.sd4_decode(codes2, meta2).float().cpu().numpy().astype(np.float64)
    assert np.array_equal(dec[:, :K] + dec[:, K:], x[[3, 1, 0, 2]])


def test_sd4_decomp_index_out_of_range_is_reported():
    x = torch.randn(8, 256, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16).cuda()
    rows = _rows_tensor([1, -1, 8, 7])
    codes2 = torch.full((4, 256), 0x5A, dtype=torch.uint8, device="cuda")
    meta2 = torch.full((4, 16), 0x1234, dtype=torch.int16, device="cuda")
    qs.qs_sd4_quant_decomp(x, 8, 256, rows, 4, codes2, meta2)
    assert qs.qs_device_error() == 5                    # QS_ERR_RANGE, then cleared
    assert qs.qs_device_error() == 0
    c = codes2.cpu().numpy()
    assert not c[1].any() and not c[2].any() and not meta2.cpu().numpy()[1:3].any()
    dec = S.decompose_rows(I.bf16_bits(x.cpu()), [1, 7])
    want_c, _ = S.pack_decomp(dec)
    assert np.array_equal(c[[0, 3]], want_c)
    # the layer call skips those rows and reports them the same way
    w = torch.randn(16, 256, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16).cuda()
    cw, mw = qs.sd4_quant(w)
    out = torch.full((8, 16), 7, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    qs.qs_sd4_linear_decomp(codes2, meta2, rows, 4, cw, mw, None, None, 8, 16, 256, out)
    assert qs.qs_device_error() == 5
    o = out.view(torch.int16).cpu().numpy()
    assert (o[[0, 2, 3, 4, 5, 6]] == 7).all() and not (o[[1, 7]] == 7).all()


def _decomp_layer(M, N, K, rows, seed, wdec, bias=True):
    d = I.make_shape(seed=seed, M=M, K=K, N=N, bits=4, outlier_factor=30.0)
    x, w = d["x"].cuda(), d["w"].cuda()
    b = d["bias"].cuda() if bias else None
    cx, mx = qs.sd4_quant(x)
    cw, mw = qs.sd4_quant(w)
    rt = _rows_tensor(rows)
    codes2, meta2 = qs.sd4_quant_decomp(x, rt)
    w8 = qs.sd4_decode_e4m3(cw, mw) if wdec else None
    out = qs.sd4_linear_decomp(cx, mx, codes2, meta2, rt, cw, mw, b, K, w_e4m3=w8)
    torch.cuda.synchronize()
    return d, out


def _check_decomp_layer(d, out, rows, K, bias=True):
    xb, wb = I.bf16_bits(d["x"]), I.bf16_bits(d["w"])
    bb = I.bf16_bits(d["bias"]) if bias else None
    r = S.linear_sd4_decomp(xb, wb, bb, rows, exact=False)
    got_bits = out.view(torch.int16).cpu().numpy().view(np.uint16)
    got = O.bf16_bits_to_f32(got_bits).astype(np.float64)
    b = O.bf16_bits_to_f32(bb).astype(np.float64) if bias else 0.0
    M = got.shape[0]
    # binary32 accumulation of exact products: at most (terms) 2^-23 sum|products|
    # (2K terms on a decomposed row: x_hat and delta_hat separately), plus one
    # bf16 ulp of the result
    absw = np.abs(r["w_hat"]).T
    S_abs = np.abs(r["x_hat"]) @ absw
    terms = np.full((M, 1), float(K))
    rows_u = np.unique(rows)
    dec = r["decomp"]
    first = {int(v): i for i, v in reversed(list(enumerate(rows)))}
    sel = np.array([first[int(m)] for m in rows_u])
    S_abs[rows_u] = (np.abs(dec["x_hat"][sel]) @ absw) + (np.abs(dec["d_hat"][sel]) @ absw)
    terms[rows_u] = 2.0 * K
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(got), 2.0 ** -126))) - 7)
    allowed = terms * 2.0 ** -23 * S_abs + ulp
    err = np.abs(got - (r["y"] + b))
    assert (err <= allowed).all(), f"max excess {np.max(err - allowed)}"
    same = float((got_bits == r["out"]).mean())
    assert same > 0.99, f"only {same:.4f} of outputs bit-identical to the oracle"
    # the decomposition moved the salient rows toward the unquantised product
    xf = O.bf16_bits_to_f32(xb).astype(np.float64)
    wf = O.bf16_bits_to_f32(wb).astype(np.float64)
    ref = xf[rows_u] @ wf.T
    plain = S.linear_sd4(xb, wb, bb, exact=False)["y"][rows_u]
    assert np.linalg.norm(r["y"][rows_u] - ref) < np.linalg.norm(plain - ref)


@pytest.mark.parametrize("wdec", [False, True])
@pytest.mark.parametrize("M,N,K", [(127, 272, 256), (300, 768, 768), (513, 528, 1280)])
def test_sd4_linear_decomp_matches_oracle(M, N, K, wdec):
    rng = np.random.default_rng(M + N)
    rows = sorted(set(rng.choice(M, max(1, M // 8), replace=False).tolist()) | {0, M - 1})
    rows = rows + rows[:3]                   # repeated indices write the same values
    rng.shuffle(rows)
    d, out = _decomp_layer(M, N, K, rows, seed=M + 2 * N, wdec=wdec)
    _check_decomp_layer(d, out, rows, K)


def test_sd4_linear_decomp_single_row_no_bias_and_forms_agree():
    rows = [5]
    d, out = _decomp_layer(64, 272, 512, rows, seed=9, wdec=False, bias=False)
    _check_decomp_layer(d, out, rows, 512, bias=False)
    _, out2 = _decomp_layer(64, 272, 512, rows, seed=9, wdec=True, bias=False)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


def test_sd4_output_only_16_byte_aligned():
    """16-byte (not 32-byte) aligned outputs take the 16-byte store path."""
    M, N, K = 200, 400, 512
    d, dev, out = _layer(M, N, K, seed=41)
    cx, mx, cw, mw = dev
    x8, mx8 = qs.sd4_quant_e4m3(d["x"].cuda())
    w8 = qs.sd4_decode_e4m3(cw, mw)
    for fn in ("codes", "e4m3"):
        buf = torch.empty(M * N + 8, dtype=torch.bfloat16, device="cuda")
        o = buf[8:].view(M, N)
        assert o.data_ptr() % 32 == 16
        if fn == "codes":
            qs.qs_sd4_linear(cx, mx, cw, mw, d["bias"].cuda(), M, N, K, o)
        else:
            qs.qs_sd4_linear_e4m3(x8, mx8, w8, mw, d["bias"].cuda(), M, N, K, o)
        torch.cuda.synchronize()
        assert torch.equal(o.view(torch.int16), out.view(torch.int16)), fn


def _tiles_want(e, rows, K, weights):
    """The scale tiles from the oracle's block exponents, by the layout the
    header states (group of 128 / 192 rows padded to 128 / 256, 512-byte
    blocks, row r and block j at 512 (r / 128) + 16 (r % 32) + 4 ((r % 128) / 32) + j)."""
    group, slots = (192, 256) if weights else (128, 128)
    groups = 2 * -(-rows // 384) if weights else -(-rows // 128)
    kbs = K // 128
    out = np.zeros(groups * kbs * slots * 4, np.uint8)
    for row in range(rows):
        g, r = divmod(row, group)
        for kb in range(kbs):
            base = (g * kbs + kb) * slots * 4 + 512 * (r // 128) + 16 * (r % 32) + 4 * ((r % 128) // 32)
            for j in range(4):
                out[base + j] = (int(e[row, 4 * kb + j]) + 127) & 0xFF
    return out


@pytest.mark.parametrize("rows,K,weights", [(1, 256, 0), (129, 512, 0), (300, 768, 0),
                                            (16, 256, 1), (385, 512, 1), (200, 1280, 1)])
def test_sd4_scale_tiles_layout(rows, K, weights):
    d = I.make_shape(seed=rows + K + weights, M=rows, K=K, N=16, bits=4, outlier_factor=30.0)
    _, meta = qs.sd4_quant(d["x"].cuda())
    tiles = qs.sd4_scale_tiles(meta, bool(weights))
    torch.cuda.synchronize()
    _, e, _ = S.quantize_rows(I.bf16_bits(d["x"]))
    assert tiles.numel() == qs.qs_sd4_scale_tiles_bytes(rows, K, weights)
    assert np.array_equal(tiles.cpu().numpy(), _tiles_want(e, rows, K, weights))


@pytest.mark.parametrize("M,N,K", [(127, 272, 256), (300, 768, 768), (513, 528, 1280),
                                   (1, 16, 256), (129, 2320, 512), (4097, 2320, 256)])
def test_sd4_linear_e4m3_tiles_identical(M, N, K):
    """Scales loaded as pre-arranged tiles: bit-identical to the e4m3 GEMM
    that converts block words in the kernel (and so to the codes form, which
    the tests above compare with the oracle)."""
    d = I.make_shape(seed=7 * M + N, M=M, K=K, N=N, bits=4, outlier_factor=30.0)
    x, w, b = d["x"].cuda(), d["w"].cuda(), d["bias"].cuda()
    x8, mx = qs.sd4_quant_e4m3(x)
    cw, mw = qs.sd4_quant(w)
    w8 = qs.sd4_decode_e4m3(cw, mw)
    out8 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    qs.qs_sd4_linear_e4m3(x8, mx, w8, mw, b, M, N, K, out8)
    outt = torch.full((M, N), 3, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    qs.qs_sd4_linear_e4m3_tiles(x8, qs.sd4_scale_tiles(mx, False), w8,
                                qs.sd4_scale_tiles(mw, True), b, M, N, K, outt)
    torch.cuda.synchronize()
    assert qs.qs_device_error() == 0
    assert torch.equal(outt.view(torch.int16), out8.view(torch.int16))
