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
def test_sd4_linear_with_decoded_weights_is_identical(M, N, K):
    d, dev, out = _layer(M, N, K, seed=3 * M + N)
    cx, mx, cw, mw = dev
    wdec = qs.sd4_decode(cw, mw)
    out2 = torch.empty_like(out)
    qs.qs_sd4_linear_wdec(cx, mx, wdec, d["bias"].cuda(), M, N, K, out2)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
