"""GPU parity of bounded-init grid refinement (DVD-Quant "Resumen técnico"
§2.A) and the asymmetric-weight layer through the C ABI, against the oracle.

Bar: packed codes, scales, zero-point offsets, per-token code sums and int32
accumulators bit-identical; bf16 outputs bit-identical (within 1 ulp is the
stated bar; the epilogue's arithmetic is the oracle's order, so they match)."""

import numpy as np
import pytest
import torch

import bit_quantized_linear_hadamard_b200 as qs
from bit_quantized_linear_hadamard_b200 import build as qs_build
from bit_quantized_linear_hadamard_b200 import inputs as I
from oracle import bgr_oracle as B
from oracle import qs_oracle as O

pytestmark = pytest.mark.gpu
J, T = B.BGR_DEFAULT_CANDIDATES, B.BGR_DEFAULT_ITERATIONS


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    qs_build.build()
    qs.load()
    yield
    assert qs.qs_device_error() == 0, "a kernel reported a bounded-wait timeout"


def bits16(t):
    return I.bf16_bits(t.cpu())


def check_pack(w, bits, cand=J, iters=T, flags=0):
    wp, ws, wo = qs.pack_weights_bgr(w.cuda(), bits, cand, iters, flags)
    torch.cuda.synchronize()
    s, sw, off = B.pack_weights_bgr(bits16(w), bits, cand, iters,
                                    rotate=not (flags & qs.QS_FLAG_NO_ROTATE))
    assert np.array_equal(ws.cpu().numpy().view(np.uint32), sw.view(np.uint32)), "scales"
    assert np.array_equal(wo.cpu().numpy(), off), "offsets"
    got, want = wp.cpu().numpy(), O.pack(s, bits)
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        raise AssertionError(f"codes differ at {len(bad)} bytes, first {bad[:5].tolist()}")
    return wp, ws, wo


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("N,K", [(16, 128), (48, 640), (33, 3072), (5, 13824)])
def test_pack_weights_bgr_bit_exact(N, K, bits):
    d = I.make_shape(seed=N + K + bits, M=1, K=K, N=N, bits=bits, sigma_w=0.02)
    w = d["w"].clone()
    w[0, :: max(1, K // 7)] *= 30  # a row with outliers
    check_pack(w, bits)


@pytest.mark.parametrize("bits", [4, 8])
def test_pack_weights_bgr_edge_rows_and_settings(bits):
    w = (torch.randn(8, 256, generator=torch.Generator().manual_seed(3)) * 0.02)
    w[1] = 0.0                      # zero row: one level
    w[2] = 0.5                      # constant row (after rotation: one nonzero per block)
    w[3, 5] = 4.0                   # one large outlier
    w[4] = torch.linspace(-1, 1, 256)
    w = w.to(torch.bfloat16)
    for cand, iters in ((1, 0), (2, 1), (J, T), (256, 3)):
        check_pack(w, bits, cand, iters)
    check_pack(w, bits, flags=qs.QS_FLAG_NO_ROTATE)


@pytest.mark.parametrize("bits", [4, 6, 8])
@pytest.mark.parametrize("M,K", [(1, 128), (129, 640), (33, 5120), (17, 13824), (3, 16512)])
def test_quant_act_rowsum(M, K, bits):
    d = I.make_shape(seed=5 * M + K, M=M, K=K, N=16, bits=bits, outlier_factor=50.0)
    x = d["x"].cuda()
    for alpha in (1.0, 0.9, 0.003):
        xp, xs, xr = qs.quant_act_rowsum(x, bits, alpha)
        torch.cuda.synchronize()
        q, s = O.quant_act(bits16(d["x"]), bits, alpha)
        assert np.array_equal(xp.cpu().numpy(), O.pack(q, bits))
        assert np.array_equal(xs.cpu().numpy().view(np.uint32), s.view(np.uint32))
        assert np.array_equal(xr.cpu().numpy().astype(np.int64), B.code_rowsums(q))


GEMM_SHAPES = [(256, 512, 512), (1, 16, 128), (127, 272, 256), (300, 768, 640),
               (513, 528, 1152)]


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_qgemm_s32_asym_on_oracle_codes(M, N, K, bits):
    rng = np.random.default_rng(M + 3 * N + K + bits)
    half, qmax = 1 << (bits - 1), O.QMAX[bits]
    qa = rng.integers(-qmax, qmax + 1, (M, K)).astype(np.int8)
    s = rng.integers(-half, half, (N, K)).astype(np.int8)
    off = rng.integers(half - (2 * half - 1), half + 1, N).astype(np.int32)
    rs = B.code_rowsums(qa).astype(np.int32)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    qs.qs_qgemm_s32_asym(torch.from_numpy(O.pack(qa, bits)).cuda(), torch.from_numpy(rs).cuda(),
                         torch.from_numpy(O.pack(s, bits)).cuda(), torch.from_numpy(off).cuda(),
                         M, N, K, bits, acc)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), B.asym_accumulators(qa, s, off))


def run_bgr_layer(d, bits, alpha):
    x, w, b = d["x"].cuda(), d["w"].cuda(), d["bias"].cuda()
    wp, ws, wo = qs.pack_weights_bgr(w, bits, J, T)
    xp, xs, xr = qs.quant_act_rowsum(x, bits, alpha)
    M, K = x.shape
    N = w.shape[0]
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    qs.qs_qlinear_asym(xp, xs, xr, wp, ws, wo, b, M, N, K, bits, out)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    qs.qs_qgemm_s32_asym(xp, xr, wp, wo, M, N, K, bits, acc)
    torch.cuda.synchronize()
    return {"out": out, "acc": acc, "wp": wp, "ws": ws, "wo": wo, "xr": xr}


@pytest.mark.parametrize("bits,alpha", [(4, 1.0), (4, 0.9), (8, 1.0)])
@pytest.mark.parametrize("M,N,K", GEMM_SHAPES[:4])
def test_qlinear_bgr_matches_oracle(M, N, K, bits, alpha):
    d = I.make_shape(seed=M + N + K + 1, M=M, K=K, N=N, bits=bits, alpha=alpha,
                     outlier_factor=50.0)
    g = run_bgr_layer(d, bits, alpha)
    r = B.qlinear_bgr(bits16(d["x"]), bits16(d["w"]), bits16(d["bias"]), bits, alpha, J, T)
    assert np.array_equal(g["wp"].cpu().numpy(), r["wp"])
    assert np.array_equal(g["xr"].cpu().numpy().astype(np.int64), r["rowsum"])
    assert np.array_equal(g["acc"].cpu().numpy().astype(np.int64), r["acc"])
    got = g["out"].view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, r["out"])


@pytest.mark.parametrize("bits", [4, 8])
def test_linear_bgr_one_call(bits):
    M, N, K, alpha = 300, 768, 640, 0.9
    d = I.make_shape(seed=77 + bits, M=M, K=K, N=N, bits=bits, alpha=alpha, outlier_factor=50.0)
    g = run_bgr_layer(d, bits, alpha)
    need = qs.qs_linear_bgr_workspace_bytes(M, K, bits)
    ws = torch.full((need,), 0x3C, dtype=torch.uint8, device="cuda")  # dirty scratch
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    qs.qs_linear_bgr(d["x"].cuda(), M, K, alpha, g["wp"], g["ws"], g["wo"], d["bias"].cuda(), N,
                     bits, ws, need, out)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), g["out"].view(torch.int16))
