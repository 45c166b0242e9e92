"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bar (stated by the layer's targets): packed codes, scales and int32
accumulators bit-identical; bf16 outputs within 1 bf16 ulp (ordered bit
patterns).  Inputs are the seeded synthetic tensors; no expected value comes
from the CUDA path.  The full-size configurations, in the benchmark's launch
configuration, are compared element by element in test_gpu_full_size.py.
"""

import os

import numpy as np
import pytest
import torch

import bit_quantized_linear_hadamard_b200 as qs
from bit_quantized_linear_hadamard_b200 import build as qs_build
from bit_quantized_linear_hadamard_b200 import inputs as I
from oracle import qs_oracle as O

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


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


def ordered(b):
    b = np.asarray(b, dtype=np.int32)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def assert_within_1ulp(got_bits, want_bits, what=""):
    d = np.abs(ordered(got_bits) - ordered(want_bits))
    assert d.max(initial=0) <= 1, f"{what}: max bf16 ulp distance {d.max()} at {np.argmax(d)}"
    return float((d == 0).mean()) if d.size else 1.0


def gpu_quant(x, bits, alpha, flags=0):
    xp, xs = qs.quant_act(x.cuda(), bits, alpha, flags)
    torch.cuda.synchronize()
    return xp.cpu().numpy(), xs.cpu().numpy()


def gpu_pack(w, bits, flags=0):
    wp, ws = qs.pack_weights(w.cuda(), bits, flags)
    torch.cuda.synchronize()
    return wp.cpu().numpy(), ws.cpu().numpy()


def check_quant(x, bits, alpha, flags=0):
    xp, xs = gpu_quant(x, bits, alpha, flags)
    q, s = O.quant_act(bits16(x), bits, alpha, rotate=not (flags & qs.QS_FLAG_NO_ROTATE))
    assert np.array_equal(xs.view(np.uint32), s.view(np.uint32)), "scales differ"
    want = O.pack(q, bits)
    if not np.array_equal(xp, want):
        bad = np.argwhere(xp != want)
        raise AssertionError(f"packed codes differ at {len(bad)} bytes, first {bad[:5].tolist()}")


# --------------------------------------------------------------------------- rotate-quantize

QUANT_SHAPES = [(1, 128), (3, 256), (129, 640), (64, 3072), (33, 5120), (17, 13824),
                (5, 16384), (3, 16512), (2, 65536)]


@pytest.mark.parametrize("bits", [4, 6, 8])
@pytest.mark.parametrize("M,K", QUANT_SHAPES)
def test_quant_act_bit_exact(M, K, bits):
    d = I.make_shape(seed=100 + M + K, M=M, K=K, N=16, bits=bits, outlier_factor=50.0)
    for alpha in (1.0, 0.9):
        check_quant(d["x"], bits, alpha)


def test_quant_act_tiny_config():
    d = I.make_layer(I.TINY)
    check_quant(d["x"], 4, 1.0)


def test_quant_ties_without_rotation():
    with open(os.path.join(GOLDEN, "rne_ties_w4.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    x = torch.zeros(2, 128)
    want = np.zeros((2, 128), np.int8)
    for r, c, v, q in rows:
        x[int(r), int(c)] = float(v)
        want[int(r), int(c)] = int(q)
    xp, xs = gpu_quant(x.to(torch.bfloat16), 4, 1.0, qs.QS_FLAG_NO_ROTATE)
    assert xs.tolist() == [1.0, 0.5]
    assert np.array_equal(O.unpack(xp, 4), want)


def test_quant_rounds_the_exact_product():
    # rows where fl(u*inv) is a .5 tie but the exact u*inv is not (see the oracle
    # pin): the kernel's single rounding must follow the exact product
    from test_oracle_pins import double_rounding_rows
    rows = double_rounding_rows()
    x = torch.zeros(len(rows), 128)
    for i, (A, v, _) in enumerate(rows):
        x[i, 0], x[i, 1] = float(A), float(v)
    check_quant(x.to(torch.bfloat16), 8, 1.0, qs.QS_FLAG_NO_ROTATE)


def test_quant_zero_tiny_and_constant_rows():
    x = torch.zeros(6, 512)
    x[1] = 1e-38            # binary32 subnormal range after rotation
    x[2, 7] = -3.0
    x[3] = 2.5              # constant row: one nonzero per Hadamard block
    x[4, ::3] = 1e30
    x[5] = torch.linspace(-4, 4, 512)
    xb = x.to(torch.bfloat16)
    for bits in (4, 6, 8):
        for alpha in (1.0, 0.5, 1e-3):
            check_quant(xb, bits, alpha)


@pytest.mark.parametrize("bits", [4, 6, 8])
@pytest.mark.parametrize("alpha", [1.0 / 256, 1.0 / 256 * 0.999, 0.02])
def test_quant_small_alpha_heavy_clipping(bits, alpha):
    # most codes clip; 1/256 is the smallest alpha whose unclamped codes still
    # fit 16 bits (qmax/alpha <= 32512), just below it the float clamp is used
    d = I.make_shape(seed=77, M=40, K=1024, N=16, bits=bits, outlier_factor=100.0)
    check_quant(d["x"], bits, alpha)


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_pack_weights_bit_exact(bits):
    d = I.make_layer(I.TINY)
    wp, ws = gpu_pack(d["w"], bits)
    q, s = O.pack_weights(bits16(d["w"]), bits)
    assert np.array_equal(ws.view(np.uint32), s.view(np.uint32))
    assert np.array_equal(wp, O.pack(q, bits))
    wp, ws = gpu_pack(d["w"], bits, qs.QS_FLAG_NO_ROTATE)
    q, s = O.pack_weights(bits16(d["w"]), bits, rotate=False)
    assert np.array_equal(ws.view(np.uint32), s.view(np.uint32))
    assert np.array_equal(wp, O.pack(q, bits))


# --------------------------------------------------------------------------- integer GEMM

GEMM_SHAPES = [(256, 512, 512), (1, 16, 128), (127, 272, 256), (129, 256, 384),
               (300, 768, 640), (64, 16, 1024), (513, 528, 1152), (200, 1040, 128)]


def _codes(rng, shape, bits):
    qm = O.QMAX[bits]
    return rng.integers(-qm, qm + 1, size=shape).astype(np.int8)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_qgemm_s32_bit_exact_on_oracle_codes(M, N, K, bits):
    rng = np.random.default_rng(M * 7 + N * 3 + K + bits)
    qa, qw = _codes(rng, (M, K), bits), _codes(rng, (N, K), bits)
    xp = torch.from_numpy(O.pack(qa, bits)).cuda()
    wp = torch.from_numpy(O.pack(qw, bits)).cuda()
    acc = qs.qgemm_s32(xp, wp, bits, K)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), O.int_gemm(qa, qw))


@pytest.mark.parametrize("bits", [4, 8])
def test_qgemm_s32_extreme_codes_at_max_k(bits):
    K, qm = 65536, O.QMAX[bits]
    qa = np.full((3, K), qm, np.int8)
    qa[1] = -qm
    qa[2, ::2] = -qm
    qw = np.full((16, K), -qm, np.int8)
    qw[5] = qm
    acc = qs.qgemm_s32(torch.from_numpy(O.pack(qa, bits)).cuda(),
                       torch.from_numpy(O.pack(qw, bits)).cuda(), bits, K)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), O.int_gemm(qa, qw))


# mixed code widths (x, W): W4A8, W4A6, and the other pairings the kernel serves
MIXED = [(8, 4), (6, 4), (4, 8), (6, 6), (6, 8)]


@pytest.mark.parametrize("bx,bw", MIXED)
@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_qgemm_s32_mixed_bit_exact_on_oracle_codes(M, N, K, bx, bw):
    rng = np.random.default_rng(M * 5 + N * 11 + K + 10 * bx + bw)
    qa, qw = _codes(rng, (M, K), bx), _codes(rng, (N, K), bw)
    xp = torch.from_numpy(O.pack(qa, bx)).cuda()
    wp = torch.from_numpy(O.pack(qw, bw)).cuda()
    acc = qs.qgemm_s32(xp, wp, bx, K, bits_w=bw)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), O.int_gemm(qa, qw))


@pytest.mark.parametrize("bx,bw", [(8, 4), (4, 8)])
def test_qgemm_s32_mixed_extreme_codes_at_max_k(bx, bw):
    # 127 * 7 * 65536 with the 4-bit side widened to 16 q: the hardware sum
    # 16 * 127 * 7 * 65536 still fits int32
    K = 65536
    qa = np.full((3, K), O.QMAX[bx], np.int8)
    qa[1] = -O.QMAX[bx]
    qa[2, ::2] = -O.QMAX[bx]
    qw = np.full((16, K), -O.QMAX[bw], np.int8)
    qw[5] = O.QMAX[bw]
    acc = qs.qgemm_s32(torch.from_numpy(O.pack(qa, bx)).cuda(),
                       torch.from_numpy(O.pack(qw, bw)).cuda(), bx, K, bits_w=bw)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), O.int_gemm(qa, qw))


# --------------------------------------------------------------------------- whole layer

def run_layer(d, bits, alpha, bias=True, bits_x=None, x_flags=0):
    """bits: the weights' code width; bits_x: the activations' (default bits);
    x_flags: their storage (QS_FLAG_BYTE_CODES: 4-bit codes one per byte)."""
    bx = bits if bits_x is None else bits_x
    sx = qs.storage_bits(bx, x_flags)
    x, w, b = d["x"].cuda(), d["w"].cuda(), d["bias"].cuda() if bias else None
    wp, ws = qs.pack_weights(w, bits)
    xp, xs = qs.quant_act(x, bx, alpha, x_flags)
    out = qs.qlinear(xp, xs, wp, ws, b, sx, x.shape[1], bits_w=bits)
    acc = qs.qgemm_s32(xp, wp, sx, x.shape[1], bits_w=bits)
    torch.cuda.synchronize()
    return {"out": out, "acc": acc, "xp": xp, "xs": xs, "wp": wp, "ws": ws}


@pytest.mark.parametrize("bits,alpha", [(4, 1.0), (4, 0.9), (8, 1.0)])
@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_qlinear_matches_oracle(M, N, K, bits, alpha):
    d = I.make_shape(seed=M + N + K, M=M, K=K, N=N, bits=bits, alpha=alpha, outlier_factor=50.0)
    g = run_layer(d, bits, alpha)
    r = O.qlinear(bits16(d["x"]), bits16(d["w"]), bits16(d["bias"]), bits, alpha)
    assert np.array_equal(g["xp"].cpu().numpy(), r["xp"])
    assert np.array_equal(g["wp"].cpu().numpy(), r["wp"])
    assert np.array_equal(g["acc"].cpu().numpy().astype(np.int64), r["acc"])
    got = g["out"].view(torch.int16).cpu().numpy().view(np.uint16)
    exact = assert_within_1ulp(got, r["out"], f"{M}x{N}x{K} w{bits}")
    assert exact == 1.0, f"only {exact:.6f} of outputs bit-identical"


@pytest.mark.parametrize("bx,bw,alpha", [(8, 4, 1.0), (8, 4, 0.9), (6, 4, 0.9), (4, 8, 1.0),
                                         (6, 6, 1.0)])
@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_qlinear_mixed_matches_oracle(M, N, K, bx, bw, alpha):
    d = I.make_shape(seed=M + 2 * N + K, M=M, K=K, N=N, bits=bw, alpha=alpha, outlier_factor=50.0,
                     bits_x=bx)
    g = run_layer(d, bw, alpha, bits_x=bx)
    r = O.qlinear_mixed(bits16(d["x"]), bits16(d["w"]), bits16(d["bias"]), bx, bw, alpha)
    assert np.array_equal(g["xp"].cpu().numpy(), r["xp"])
    assert np.array_equal(g["wp"].cpu().numpy(), r["wp"])
    assert np.array_equal(g["acc"].cpu().numpy().astype(np.int64), r["acc"])
    got = g["out"].view(torch.int16).cpu().numpy().view(np.uint16)
    exact = assert_within_1ulp(got, r["out"], f"{M}x{N}x{K} a{bx}w{bw}")
    assert exact == 1.0, f"only {exact:.6f} of outputs bit-identical"


@pytest.mark.parametrize("bx,bw", [(8, 4), (6, 4)])
def test_linear_mixed_one_call(bx, bw):
    M, N, K, alpha = 300, 768, 640, 0.9
    d = I.make_shape(seed=31 + bx, M=M, K=K, N=N, bits=bw, alpha=alpha, outlier_factor=50.0,
                     bits_x=bx)
    g = run_layer(d, bw, alpha, bits_x=bx)
    need = qs.qs_linear_workspace_bytes(M, K, bx)
    ws = torch.full((need,), 0x5A, dtype=torch.uint8, device="cuda")
    out = qs.linear(d["x"].cuda(), g["wp"], g["ws"], d["bias"].cuda(), bx, alpha, workspace=ws,
                    bits_w=bw)
    layer = qs.QuantLinear(d["w"].cuda(), d["bias"].cuda(), bw, alpha, bits_x=bx)
    out2 = layer(d["x"].cuda())
    torch.cuda.synchronize()
    want = g["out"].view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), want)
    assert np.array_equal(out2.view(torch.int16).cpu().numpy().view(np.uint16), want)
    r = O.qlinear_mixed(bits16(d["x"]), bits16(d["w"]), bits16(d["bias"]), bx, bw, alpha)
    assert np.array_equal(want, r["out"])


@pytest.mark.parametrize("act_codes", ["bytes", "packed"])
def test_quant_linear_layer_w4a4_both_code_layouts(act_codes):
    M, N, K, alpha = 300, 768, 640, 0.9
    d = I.make_shape(seed=37, M=M, K=K, N=N, bits=4, alpha=alpha, outlier_factor=50.0)
    layer = qs.QuantLinear(d["w"].cuda(), d["bias"].cuda(), 4, alpha, act_codes=act_codes)
    assert layer.x_flags == (qs.QS_FLAG_BYTE_CODES if act_codes == "bytes" else 0)
    out = layer(d["x"].cuda())
    out_again = layer(d["x"][:7].cuda())  # the workspace kept from the larger call
    torch.cuda.synchronize()
    r = O.qlinear(bits16(d["x"]), bits16(d["w"]), bits16(d["bias"]), 4, alpha)
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), r["out"])
    assert np.array_equal(out_again.view(torch.int16).cpu().numpy().view(np.uint16), r["out"][:7])


def test_qlinear_null_bias_and_zero_rows():
    d = I.make_shape(seed=5, M=130, K=256, N=272, bits=4)
    d["x"][3] = 0
    d["x"][129] = 0
    g = run_layer(d, 4, 1.0, bias=False)
    r = O.qlinear(bits16(d["x"]), bits16(d["w"]), None, 4, 1.0)
    got = g["out"].view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, r["out"])
    assert not got[3].any() and not got[129].any()


@pytest.mark.parametrize("bits,alpha", [(4, 0.9), (8, 1.0)])
@pytest.mark.parametrize("M,N,K", [(300, 768, 640), (1, 16, 128), (513, 528, 1152)])
def test_linear_one_call_matches_two_calls_and_oracle(M, N, K, bits, alpha):
    d = I.make_shape(seed=7 * M + K, M=M, K=K, N=N, bits=bits, alpha=alpha, outlier_factor=50.0)
    g = run_layer(d, bits, alpha)
    need = qs.qs_linear_workspace_bytes(M, K, bits)
    ws = torch.full((need,), 0xA5, dtype=torch.uint8, device="cuda")  # dirty scratch
    out = qs.linear(d["x"].cuda(), g["wp"], g["ws"], d["bias"].cuda(), bits, alpha, workspace=ws)
    torch.cuda.synchronize()
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, g["out"].view(torch.int16).cpu().numpy().view(np.uint16))
    r = O.qlinear(bits16(d["x"]), bits16(d["w"]), bits16(d["bias"]), bits, alpha)
    assert np.array_equal(got, r["out"])


def test_tiny_config_full_parity():
    d = I.make_layer(I.TINY)
    g = run_layer(d, 4, 1.0)
    r = O.qlinear(bits16(d["x"]), bits16(d["w"]), bits16(d["bias"]), 4, 1.0)
    assert np.array_equal(g["acc"].cpu().numpy().astype(np.int64), r["acc"])
    got = g["out"].view(torch.int16).cpu().numpy().view(np.uint16)
    assert assert_within_1ulp(got, r["out"], "tiny") == 1.0


def test_gelu_matches_oracle():
    x = (torch.randn(4097, generator=torch.Generator().manual_seed(9)) * 3).to(torch.bfloat16)
    y = qs.gelu(x.cuda())
    torch.cuda.synchronize()
    got = y.view(torch.int16).cpu().numpy().view(np.uint16)
    assert_within_1ulp(got, O.gelu_erf_bf16(bits16(x)), "gelu")


def test_gelu_table_path_covers_every_bf16_pattern():
    """Inputs of 2^24 elements and more take the shared-memory table kernel:
    every one of the 65536 bf16 bit patterns (tiled 256 times, plus a ragged
    tail of 5) must give the direct kernel's bits, and every finite pattern
    must be within 1 bf16 ulp of the oracle."""
    pats = np.arange(65536, dtype=np.uint16)
    direct = qs.gelu(torch.from_numpy(pats.view(np.int16)).view(torch.bfloat16).cuda())
    big = np.concatenate([np.tile(pats, 256), pats[:5]])
    tab = qs.gelu(torch.from_numpy(big.view(np.int16)).view(torch.bfloat16).cuda())
    torch.cuda.synchronize()
    d = direct.view(torch.int16).cpu().numpy().view(np.uint16)
    t = tab.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(t[:65536 * 256].reshape(256, 65536), np.broadcast_to(d, (256, 65536)))
    assert np.array_equal(t[65536 * 256:], d[:5])
    finite = (pats & 0x7F80) != 0x7F80
    assert_within_1ulp(d[finite], O.gelu_erf_bf16(pats[finite]), "gelu all patterns")


# --------------------------------------------------------------------------- multi-tile grids, in full

# (bits_x, bits_w, x_flags): packed W4A4, W4A4 with byte-stored activation
# codes (the mixed-storage kernel), W8A8 (banded tile order) and W4A8
MULTI_TILE_FORMS = [(4, 4, 0), (4, 4, qs.QS_FLAG_BYTE_CODES), (8, 8, 0), (8, 4, 0)]


@pytest.mark.parametrize("bx,bw,flags", MULTI_TILE_FORMS, ids=["w4a4", "w4a4_bytes", "w8a8", "w4a8"])
def test_multi_tile_grid_every_element(bx, bw, flags):
    """M = 4096, N = 5120, K = 5120: 16 x 10 = 160 output tiles of 256 x 512
    (16 x 20 = 320 of 256 x 256 in the 8-bit x 8-bit form) for 74 CTA pairs,
    so every pair runs several tiles (the persistent loop, the tensor-memory
    accumulators drained and reused, the operand ring wrapping many times)
    and the 8-bit x 8-bit form crosses a band edge (18 + 2 N-tiles).  Every
    code, scale, accumulator and output is compared with the oracle."""
    M, N, K, alpha = 4096, 5120, 5120, 0.9
    d = I.make_shape(seed=4096 + 10 * bx + bw, M=M, K=K, N=N, bits=bw, alpha=alpha,
                     outlier_factor=100.0, outlier_frac=0.005, sigma_w=0.015,
                     bits_x=bx if bx != bw else 0)
    g = run_layer(d, bw, alpha, bits_x=bx, x_flags=flags)
    qa, sa = O.quant_act(bits16(d["x"]), bx, alpha)
    qw, sw = O.pack_weights(bits16(d["w"]), bw)
    assert np.array_equal(g["xs"].cpu().numpy().view(np.uint32), sa.view(np.uint32))
    assert np.array_equal(g["xp"].cpu().numpy(), O.pack(qa, qs.storage_bits(bx, flags)))
    assert np.array_equal(g["ws"].cpu().numpy().view(np.uint32), sw.view(np.uint32))
    assert np.array_equal(g["wp"].cpu().numpy(), O.pack(qw, bw))
    acc = O.int_gemm_f64(qa, qw)
    assert np.array_equal(g["acc"].cpu().numpy().astype(np.int64), acc)
    want = O.epilogue(acc, sa, sw, bits16(d["bias"]))
    got = g["out"].view(torch.int16).cpu().numpy().view(np.uint16)
    assert assert_within_1ulp(got, want, "multi-tile") == 1.0


@pytest.mark.parametrize("bx,bw,flags", MULTI_TILE_FORMS, ids=["w4a4", "w4a4_bytes", "w8a8", "w4a8"])
def test_wide_tile_ragged_edges_every_element(bx, bw, flags):
    """N = 2320 = 4 x 512 + 272: the last 256 x 512 tile has a full first
    N-half and 16 columns of its second; M = 1000 ends in a ragged M-tile
    (232 rows); K = 5120 as in the Wan FFN.  Every code, scale, accumulator
    and output against the oracle."""
    M, N, K, alpha = 1000, 2320, 5120, 0.9
    d = I.make_shape(seed=2320 + 10 * bx + bw, M=M, K=K, N=N, bits=bw, alpha=alpha,
                     outlier_factor=100.0, outlier_frac=0.005, sigma_w=0.015,
                     bits_x=bx if bx != bw else 0)
    g = run_layer(d, bw, alpha, bits_x=bx, x_flags=flags)
    qa, sa = O.quant_act(bits16(d["x"]), bx, alpha)
    qw, sw = O.pack_weights(bits16(d["w"]), bw)
    assert np.array_equal(g["xs"].cpu().numpy().view(np.uint32), sa.view(np.uint32))
    assert np.array_equal(g["xp"].cpu().numpy(), O.pack(qa, qs.storage_bits(bx, flags)))
    assert np.array_equal(g["wp"].cpu().numpy(), O.pack(qw, bw))
    acc = O.int_gemm_f64(qa, qw)
    assert np.array_equal(g["acc"].cpu().numpy().astype(np.int64), acc)
    want = O.epilogue(acc, sa, sw, bits16(d["bias"]))
    got = g["out"].view(torch.int16).cpu().numpy().view(np.uint16)
    assert assert_within_1ulp(got, want, "ragged wide tile") == 1.0


def test_w8a8_band_edge_small():
    """The 8-bit x 8-bit form walks N-tiles in bands of 18: N = 5120 has 20
    N-tiles (a full band and a last band of 2), M = 300 a ragged second M-tile.
    Full int32 and bf16 parity."""
    M, N, K = 300, 5120, 256
    d = I.make_shape(seed=3005, M=M, K=K, N=N, bits=8, outlier_factor=50.0)
    g = run_layer(d, 8, 1.0)
    r = O.qlinear(bits16(d["x"]), bits16(d["w"]), bits16(d["bias"]), 8, 1.0)
    assert np.array_equal(g["acc"].cpu().numpy().astype(np.int64), r["acc"])
    got = g["out"].view(torch.int16).cpu().numpy().view(np.uint16)
    assert assert_within_1ulp(got, r["out"], "band edge") == 1.0


# --------------------------------------------------------------------------- byte-stored 4-bit codes

@pytest.mark.parametrize("M,K", [(1, 128), (129, 640), (33, 5120), (3, 16512)])
def test_quant_act_byte_codes(M, K):
    # QS_FLAG_BYTE_CODES: the same 4-bit codes, one per byte
    d = I.make_shape(seed=2 * M + K, M=M, K=K, N=16, bits=4, outlier_factor=50.0)
    for alpha in (1.0, 0.9, 0.003):
        xp, xs = qs.quant_act(d["x"].cuda(), 4, alpha, qs.QS_FLAG_BYTE_CODES)
        torch.cuda.synchronize()
        q, s = O.quant_act(bits16(d["x"]), 4, alpha)
        assert np.array_equal(xp.cpu().numpy().view(np.int8), q)
        assert np.array_equal(xs.cpu().numpy().view(np.uint32), s.view(np.uint32))


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_w4a4_with_byte_activation_codes(M, N, K):
    # W4A4 with the activation codes in bytes: the GEMM reads them as 8-bit
    # storage; codes, accumulators and outputs equal the packed W4A4 layer's
    alpha = 0.9
    d = I.make_shape(seed=M + 5 * N + K, M=M, K=K, N=N, bits=4, alpha=alpha, outlier_factor=50.0)
    x, w, b = d["x"].cuda(), d["w"].cuda(), d["bias"].cuda()
    wp, ws = qs.pack_weights(w, 4)
    xp, xs = qs.quant_act(x, 4, alpha, qs.QS_FLAG_BYTE_CODES)
    out = qs.qlinear(xp, xs, wp, ws, b, 8, K, bits_w=4)
    acc = qs.qgemm_s32(xp, wp, 8, K, bits_w=4)
    one = qs.linear(x, wp, ws, b, 4, alpha, bits_w=4, x_flags=qs.QS_FLAG_BYTE_CODES)
    torch.cuda.synchronize()
    r = O.qlinear(bits16(d["x"]), bits16(d["w"]), bits16(d["bias"]), 4, alpha)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), r["acc"])
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, r["out"])
    assert np.array_equal(one.view(torch.int16).cpu().numpy().view(np.uint16), r["out"])


@pytest.mark.parametrize("bx,bw", [(4, 4), (8, 4), (8, 8)])
def test_qlinear_output_only_16_byte_aligned(bx, bw):
    """An output only 16-byte aligned (the ABI's requirement) takes the 16-byte
    store path; a 32-byte aligned one the 32-byte path: the same values."""
    M, N, K = 300, 272, 512
    d = I.make_shape(seed=13 + bx, M=M, K=K, N=N, bits=4, bits_x=bx if bx != bw else 0)
    x, w, b = d["x"].cuda(), d["w"].cuda(), d["bias"].cuda()
    wp, ws = qs.pack_weights(w, bw)
    xp, xs = qs.quant_act(x, bx, 1.0)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    buf = torch.empty(M * N + 8, dtype=torch.bfloat16, device="cuda")
    out16 = buf[8:].view(M, N)
    assert out.data_ptr() % 32 == 0 and out16.data_ptr() % 32 == 16
    for o in (out, out16):
        qs.qs_qlinear_mixed(xp, xs, bx, wp, ws, bw, b, M, N, K, o)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out16.view(torch.int16))
    q, s = O.quant_act(I.bf16_bits(d["x"]), bx, 1.0)
    qw, sw = O.pack_weights(I.bf16_bits(d["w"]), bw)
    want = O.epilogue(O.int_gemm(q, qw), s, sw, I.bf16_bits(d["bias"]))
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), want)
