"""GPU parity of δ-guided bit switching (DVD-Quant "Resumen técnico" §2.C)
through the C ABI, against the CPU oracle.

Bar: widths chosen per step identical to the oracle's; layer outputs
bit-identical; distances within a relative 1e-12 of the exactly rounded
oracle value (the device sums in binary64 in another order: each thread adds
at most a few thousand terms, so the rounding error is below ~1e-12 relative),
and exactly equal where every sum is an exact integer.
"""

import math

import numpy as np
import pytest
import torch

import bit_quantized_linear_hadamard_b200 as qs
from bit_quantized_linear_hadamard_b200 import build as qs_build
from bit_quantized_linear_hadamard_b200 import inputs as I
from oracle import gbs_oracle as G
from oracle import qs_oracle as O

pytestmark = pytest.mark.gpu
REL_TOL = 1e-12


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    qs_build.build()
    qs.load()
    yield
    assert qs.qs_device_error() == 0, "a kernel reported a bounded-wait timeout"


def _state():
    st = torch.zeros((qs.QS_GBS_STATE_BYTES,), dtype=torch.uint8, device="cuda")
    qs.qs_gbs_reset(st)
    return st


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _bf16(x):
    return O.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def test_reset_state():
    st = _state()
    h = qs.gbs_state_host(st)
    assert h == {"acc": 0.0, "last_d": -1.0, "bits": 8, "step": 0, "blocks_done": 0}


@pytest.mark.parametrize("n", [1, 7, 8, 9, 1000, 123457, 4 * 1024 * 1024 + 3])
def test_distance_matches_oracle(n):
    rng = np.random.default_rng(n)
    a = _bf16(rng.standard_normal(n) * np.where(rng.random(n) < 0.01, 50.0, 1.0))
    b = _bf16(rng.standard_normal(n))
    st = _state()
    qs.qs_gbs_update(_dev_bf16(a), _dev_bf16(b), n, 1e300, st)
    got = qs.gbs_state_host(st)
    want = G.l1_distance(a, b)
    assert abs(got["last_d"] - want) <= REL_TOL * want, (got["last_d"], want)
    assert got["bits"] == 4 and got["step"] == 1 and got["blocks_done"] == 0


def test_distance_exact_cases():
    rng = np.random.default_rng(1)
    y = _bf16(rng.standard_normal(100003))
    y2 = _bf16(2 * O.bf16_bits_to_f32(y))
    yn = _bf16(-O.bf16_bits_to_f32(y))
    z = np.zeros_like(y)
    for cur, prev, want in ((y, y, 0.0), (y2, y, 1.0), (yn, y, 2.0), (z, y, 1.0), (z, z, 0.0),
                            (y, z, math.inf)):
        st = _state()
        qs.qs_gbs_update(_dev_bf16(cur), _dev_bf16(prev), cur.size, 1e300, st)
        assert qs.gbs_state_host(st)["last_d"] == want


def test_decisions_on_integer_outputs_are_exact():
    # integer-valued outputs: every sum is an exact integer, so distances,
    # accumulators and widths must equal the oracle's exactly
    rng = np.random.default_rng(7)
    n, T, delta = 50000, 40, 0.7
    ys = [rng.integers(-8, 9, n).astype(np.float32)]
    for t in range(1, T):
        y = ys[-1].copy()
        frac = [0.0, 0.02, 0.1, 0.3, 0.6][t % 5]
        k = int(frac * n)
        idx = rng.choice(n, k, replace=False)
        y[idx] = rng.integers(-8, 9, k)
        ys.append(y)
    bits = [_bf16(y) for y in ys]
    st = _state()
    s = G.GbsState()
    widths = []
    for t in range(T):
        prev = None if t == 0 else _dev_bf16(bits[t - 1])
        qs.qs_gbs_update(_dev_bf16(bits[t]), prev, n, delta, st)
        s = G.gbs_update(s, None if t == 0 else G.l1_distance(bits[t], bits[t - 1]), delta)
        h = qs.gbs_state_host(st)
        assert (h["acc"], h["bits"], h["step"]) == (s.acc, s.bits, s.step), t
        widths.append(h["bits"])
    assert 4 in widths and 8 in widths


def _evolving_inputs(cfg_seed, M, K, T, sigmas):
    g = torch.Generator().manual_seed(cfg_seed)
    x = torch.randn(M, K, generator=g)
    cols = torch.randperm(K, generator=g)[: max(1, K // 100)]
    x[:, cols] *= 50.0
    xs = []
    for t in range(T):
        if t:
            x = x + sigmas[t] * torch.randn(M, K, generator=g)
        xs.append(x.to(torch.bfloat16))
    return xs


def test_layer_sequence_matches_oracle():
    M, K, N, T, alpha = 300, 640, 768, 10, 0.9
    sigmas = [0, 0.02, 0.02, 0.5, 0.01, 0.01, 0.01, 0.2, 0.05, 0.0]
    xs = _evolving_inputs(5, M, K, T, sigmas)
    g = torch.Generator().manual_seed(6)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    b = (torch.randn(N, generator=g) * 0.01).to(torch.bfloat16)
    xb = [I.bf16_bits(x) for x in xs]
    # pick delta from the oracle's own trace so that no accumulator lies
    # within 1e-9 of it (where rounding order could flip the decision)
    d_all = G.gbs_run(xb, I.bf16_bits(w), I.bf16_bits(b), alpha, 1e300)["d"]
    delta = 0.5 * sorted(d for d in d_all if d)[len(d_all) // 2] * 3
    r = G.gbs_run(xb, I.bf16_bits(w), I.bf16_bits(b), alpha, delta)
    acc = 0.0
    for s, d in zip(r["states"], r["d"]):
        if d is not None:
            assert abs(acc + d - delta) > 1e-9 * delta, "delta too close to an accumulator"
        acc = s.acc
    assert 4 in r["bits"] and r["bits"].count(8) >= 2, r["bits"]

    layer = qs.GbsLinear(w.cuda(), b.cuda(), delta, alpha)
    for t, x in enumerate(xs):
        assert qs.gbs_state_host(layer.state)["bits"] == r["bits"][t], t
        y = layer(x.cuda())
        torch.cuda.synchronize()
        got = y.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got, r["out"][t]), f"step {t} at {r['bits'][t]} bits"
        h = qs.gbs_state_host(layer.state)
        if r["d"][t] is None:
            assert h["last_d"] == -1.0
        else:
            assert abs(h["last_d"] - r["d"][t]) <= REL_TOL * r["d"][t]
        assert h["bits"] == r["states"][t].bits and h["step"] == t + 1


@pytest.mark.parametrize("width", [4, 8])
def test_gated_layer_runs_only_the_selected_width(width):
    d = I.make_shape(seed=9, M=129, K=384, N=272, bits=4, outlier_factor=30.0)
    x, w, b = d["x"].cuda(), d["w"].cuda(), d["bias"].cuda()
    layer = qs.GbsLinear(w, b, delta=1e300 if width == 4 else 0.0)
    if width == 4:  # one update without a previous output moves the state to 4 bits
        qs.qs_gbs_update(torch.zeros(16, dtype=torch.bfloat16, device="cuda"), None, 16, 1e300,
                         layer.state)
    assert qs.gbs_state_host(layer.state)["bits"] == width
    out = torch.full((129, 272), float("nan"), dtype=torch.bfloat16, device="cuda")
    qs.qs_linear_gbs(x, 129, 384, 1.0, layer.w4, layer.s4, layer.w8, layer.s8, b, 272,
                     layer.state, torch.empty(qs.qs_linear_workspace_bytes(129, 384, 8),
                                              dtype=torch.uint8, device="cuda"),
                     qs.qs_linear_workspace_bytes(129, 384, 8), out)
    torch.cuda.synchronize()
    want = O.qlinear(I.bf16_bits(d["x"]), I.bf16_bits(d["w"]), I.bf16_bits(d["bias"]), width,
                     1.0)["out"]
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), want)


@pytest.mark.slow
def test_full_size_distance_property():
    # Wan-14B FFN up-projection output (32760 x 13824 bf16): the device distance
    # against a chunked binary64 sum on the host
    cfg = I.WAN_FFN
    d = I.make_layer(cfg)
    layer = qs.GbsLinear(d["w"].cuda(), d["bias"].cuda(), delta=1e300, alpha=cfg.alpha)
    x0 = d["x"].cuda()
    y0 = layer(x0).clone()
    g = torch.Generator(device="cpu").manual_seed(12)
    x1 = (d["x"].float() + 0.05 * torch.randn(d["x"].shape, generator=g)).to(torch.bfloat16)
    y1 = layer(x1.cuda())
    torch.cuda.synchronize()
    h = qs.gbs_state_host(layer.state)
    a = y1.view(torch.int16).cpu().numpy().view(np.uint16).ravel()
    b = y0.view(torch.int16).cpu().numpy().view(np.uint16).ravel()
    num = den = 0.0
    for i in range(0, a.size, 1 << 24):  # binary64 pairwise sums, chunk by chunk
        diff, ref = G.l1_terms(a[i:i + (1 << 24)], b[i:i + (1 << 24)])
        num += float(np.sum(diff))
        den += float(np.sum(ref))
    want = num / den
    assert abs(h["last_d"] - want) <= 1e-9 * want, (h["last_d"], want)
    assert h["step"] == 2 and h["bits"] == 4
