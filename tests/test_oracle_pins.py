"""Pins of the CPU oracle against what the mathematics and the pages fix.

None of these re-types the oracle's own formulas: each compares it with an
independent definition (the Sylvester closed form of the Hadamard entries,
exact integer arithmetic, Parseval, rotation invariance of the unquantised
product, hand-derived worked rows under tests/golden/, brute-force loops,
torch's own bf16 rounding).  ``test_oracle_mutants.py`` plants plausible
mistakes in the oracle and checks that at least one pin here catches each.
"""

import math
import os
import struct

import numpy as np
import pytest
import torch

import oracle
from oracle import qs_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(a):
    return O.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def _closed_form_h(n=128):
    """Sylvester Hadamard entries from the popcount closed form (pure Python)."""
    return np.array([[(-1) ** bin(i & j).count("1") for j in range(n)] for i in range(n)],
                    dtype=np.int64)


def _load_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append(line.split())
    return rows


# --------------------------------------------------------------------------- Hadamard

def pin_fwht_unit_vectors(o=O):
    h = _closed_form_h()
    eye = np.eye(128, dtype=np.float32)
    u = o.fwht128_blocks(eye)
    assert np.array_equal(u.astype(np.int64), h), "FWHT(e_i) must be row i of the Sylvester matrix"


def pin_fwht_involution(o=O):
    h = _closed_form_h().astype(np.float32)
    hh = o.fwht128_blocks(h)  # rows of H transformed: H·H
    assert np.array_equal(hh, 128 * np.eye(128, dtype=np.float32)), "H·H must be 128·I"


def pin_fwht_exact_integers(o=O):
    rng = np.random.default_rng(11)
    x = rng.integers(-8, 9, size=(6, 512)).astype(np.int64)
    h = _closed_form_h()
    want = np.concatenate([x[:, b * 128:(b + 1) * 128] @ h for b in range(4)], axis=1)
    got = o.fwht128_blocks(x.astype(np.float32))
    assert np.array_equal(got.astype(np.int64), want), "block FWHT of small integers is exact"


def pin_parseval(o=O):
    rng = np.random.default_rng(12)
    x = rng.standard_normal((8, 384)).astype(np.float32)
    u = o.fwht128_blocks(x).astype(np.float64)
    xb = x.astype(np.float64).reshape(8, 3, 128)
    ub = u.reshape(8, 3, 128)
    lhs = (ub ** 2).sum(-1)
    rhs = 128.0 * (xb ** 2).sum(-1)
    assert np.allclose(lhs, rhs, rtol=1e-5), "Parseval per 128-block"


def pin_rotation_invariance(o=O):
    # The unquantised rotated product (x R)(W R)^T equals x W^T: relative Frobenius
    # error at most 1e-4 with the rotation computed in binary32.
    rng = np.random.default_rng(13)
    x = _bf16(rng.standard_normal((64, 512)) * np.where(rng.random(512) < 0.02, 30.0, 1.0))
    w = _bf16(rng.standard_normal((96, 512)) * 0.02)
    xf = O.bf16_bits_to_f32(x)
    wf = O.bf16_bits_to_f32(w)
    inv = np.float32(1.0 / math.sqrt(128.0))
    xr = (o.fwht128_blocks(xf) * inv).astype(np.float64)
    wr = (o.fwht128_blocks(wf) * inv).astype(np.float64)
    ref = xf.astype(np.float64) @ wf.astype(np.float64).T
    got = xr @ wr.T
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel <= 1e-4, rel


# --------------------------------------------------------------------------- quantiser

def pin_quant_error_bound(o=O):
    rng = np.random.default_rng(14)
    x = _bf16(rng.standard_normal((32, 640)) * np.where(rng.random(640) < 0.01, 50.0, 1.0))
    for bits in (4, 6, 8):
        for alpha in (1.0, 0.9, 0.5):
            q, s = o.quant_act(x, bits, alpha)
            u = O.fwht128_blocks(O.bf16_bits_to_f32(x)).astype(np.float64)
            qmax = O.QMAX[bits]
            s64 = s.astype(np.float64)[:, None]
            deq = q.astype(np.float64) * s64
            unclipped = np.abs(u) <= qmax * s64
            err = np.abs(u - deq)
            # r = u * fl(qmax / t) (exact product) carries 2 roundings relative to
            # u / s, each at most 2^-24 relative, and |u / s| <= qmax / alpha.
            bound = s64 / 2 + s64 * (qmax / alpha + 1) * 2.0 ** -22
            assert np.all(err[unclipped] <= np.broadcast_to(bound, err.shape)[unclipped]), (bits, alpha)
            clipped = ~unclipped
            assert np.all(np.abs(q[clipped]) == qmax), "clipped values saturate"
            assert np.all(np.sign(q[clipped]) == np.sign(u[clipped])), "with the sign of u"
            assert np.all(np.abs(q) <= qmax), "symmetric range, -qmax-1 never produced"
            want_s = np.abs(u).max(1) * alpha / qmax
            assert np.allclose(s, want_s, rtol=1e-6), "scale = alpha*amax/qmax of the rotated row"


def pin_rne_ties(o=O):
    rows = _load_rows("rne_ties_w4.txt")
    x = np.zeros((2, 128), dtype=np.float32)
    want = np.zeros((2, 128), dtype=np.int64)
    for r, c, v, q in rows:
        x[int(r), int(c)] = float(v)
        want[int(r), int(c)] = int(q)
    q, s = o.quantize_rows(_bf16(x), 4, 1.0, rotate=False)
    assert s.tolist() == [1.0, 0.5]
    assert np.array_equal(q.astype(np.int64), want)


def double_rounding_rows():
    """Rows (bf16 values, no rotation, int8, alpha = 1) that each hold an amax A in
    [128, 256) and one value u < A for which fl(u * inv) is a .5 tie while the
    exact product u * inv = u * fl(127 / A) is not: the two roundings disagree."""
    us = O.bf16_bits_to_f32(np.arange(0x3F80, 0x4380, dtype=np.uint16))
    rows = []
    for A in O.bf16_bits_to_f32(np.arange(0x4300, 0x4380, dtype=np.uint16)):
        inv = np.float32(127.0) / np.float32(A)
        u = us[us < A]
        r32 = u * inv
        tie = (r32 == np.floor(r32) + np.float32(0.5)) & (u.astype(np.float64) * float(inv) != r32)
        for v in u[tie]:
            rows.append((A, v, int(np.rint(float(v) * float(inv)))))
    return rows


def pin_exact_product_rounding(o=O):
    """The code rounds the exact product u*inv once (not fl(u*inv) then rint)."""
    rows = double_rounding_rows()
    assert len(rows) > 10, "the search must find double-rounding cases"
    x = np.zeros((len(rows), 128), np.float32)
    for i, (A, v, _) in enumerate(rows):
        x[i, 0], x[i, 1] = A, v
    q, _ = o.quant_act(_bf16(x), 8, 1.0, rotate=False)
    assert [int(t) for t in q[:, 1]] == [want for _, _, want in rows]


def pin_absmax_maps_to_qmax(o=O):
    rng = np.random.default_rng(15)
    x = _bf16(rng.standard_normal((16, 256)))
    u = O.fwht128_blocks(O.bf16_bits_to_f32(x))
    for bits in (4, 6, 8):
        q, _ = o.quant_act(x, bits, 1.0)
        idx = np.abs(u).argmax(1)
        got = q[np.arange(16), idx].astype(np.int64)
        assert np.array_equal(np.abs(got), np.full(16, O.QMAX[bits])), bits
        assert np.array_equal(np.sign(got), np.sign(u[np.arange(16), idx]).astype(np.int64))


def pin_zero_row(o=O):
    x = np.zeros((2, 256), dtype=np.uint16)
    x[1, 5] = _bf16([3.0])[0]
    w = _bf16(np.random.default_rng(16).standard_normal((8, 256)) * 0.02)
    b = _bf16(np.linspace(-0.05, 0.05, 8))
    r = o.qlinear(x, w, b, 4, 1.0)
    assert r["sa"][0] == 0 and not r["qa"][0].any()
    assert np.array_equal(r["out"][0], b), "a zero token gives exactly the bias"
    # below the zero-row threshold (alpha*amax < 2^-120) codes are 0; just above it
    # the single nonzero input spreads to +-amax everywhere and every code is +-qmax
    tiny = np.zeros((2, 128), np.float32)
    tiny[0, 3] = 2.0 ** -125
    tiny[1, 3] = 2.0 ** -110
    q, s = o.quant_act(_bf16(tiny), 4, 1.0)
    assert s[0] == 0 and not q[0].any()
    assert s[1] > 0 and np.all(np.abs(q[1]) == 7)


# --------------------------------------------------------------------------- packing

def pin_pack_golden(o=O):
    rows = _load_rows("pack_w4.txt")
    codes = np.array([[int(a), int(b)] for a, b, _ in rows], dtype=np.int8).reshape(1, -1)
    want = np.array([int(h, 16) for _, _, h in rows], dtype=np.uint8).reshape(1, -1)
    assert np.array_equal(o.pack(codes, 4), want)
    assert np.array_equal(o.unpack(want, 4), codes)


def pin_pack_roundtrip(o=O):
    rng = np.random.default_rng(17)
    for bits in (4, 8):
        qm = O.QMAX[bits]
        q = rng.integers(-qm, qm + 1, size=(5, 256)).astype(np.int8)
        p = o.pack(q, bits)
        assert p.shape == (5, 256 * bits // 8)
        assert np.array_equal(o.unpack(p, bits), q)
    q8 = np.array([[-128, -1, 0, 1, 127, -7, 7, 5]], dtype=np.int8)
    assert o.pack(q8, 8).tolist() == [[0x80, 0xFF, 0, 1, 0x7F, 0xF9, 7, 5]], "int8 is two's complement"


# --------------------------------------------------------------------------- integer GEMM

def pin_mixed_widths(o=O):
    """W4A8 / W4A6: the mixed layer equals quantising each side at its own width
    (qmax 7, 31 or 127; 6-bit codes in int8 bytes) and the exact integer product."""
    rng = np.random.default_rng(23)
    x = _bf16(rng.standard_normal((6, 256)) * np.where(rng.random(256) < 0.02, 30.0, 1.0))
    w = _bf16(rng.standard_normal((5, 256)) * 0.02)
    for bx, bw in ((8, 4), (6, 4), (4, 8)):
        r = o.qlinear_mixed(x, w, None, bx, bw, 0.9)
        # symmetric b-bit grid: qmax = 2^(b-1) - 1; clipping (alpha < 1) saturates
        # every activation row and each weight row's absmax lands on qmax
        qmax = {4: 7, 6: 31, 8: 127}
        assert (np.abs(r["qa"]).max(axis=1) == qmax[bx]).all()
        assert (np.abs(r["qw"]).max(axis=1) == qmax[bw]).all()
        assert r["xp"].shape[1] == (128 if bx == 4 else 256)
        assert r["wp"].shape[1] == (128 if bw == 4 else 256)
        brute = [[sum(int(r["qa"][m, k]) * int(r["qw"][n, k]) for k in range(256))
                  for n in range(5)] for m in range(6)]
        assert r["acc"].tolist() == brute
    q6 = np.array([[-31, -1, 0, 1, 31]], np.int8)
    assert o.pack(q6, 6).tolist() == [[0xE1, 0xFF, 0, 1, 0x1F]]


def pin_int_gemm_bruteforce(o=O):
    rng = np.random.default_rng(18)
    for bits in (4, 8):
        qm = O.QMAX[bits]
        a = rng.integers(-qm, qm + 1, size=(8, 128)).astype(np.int8)
        w = rng.integers(-qm, qm + 1, size=(8, 128)).astype(np.int8)
        want = [[sum(int(a[m, k]) * int(w[n, k]) for k in range(128)) for n in range(8)] for m in range(8)]
        assert o.int_gemm(a, w).tolist() == want
        f64 = a.astype(np.float64) @ w.astype(np.float64).T
        assert np.array_equal(o.int_gemm(a, w).astype(np.float64), f64)


def pin_int_gemm_f64_exact(o=O):
    """The binary64-BLAS accumulators (used for full-size parity) equal exact
    integer sums: brute-force Python loops on 8 x 8 x 128, and at K = 65536
    with extreme codes, where sums reach 127^2 K ~ 1.06e9 (a binary32 product
    would round there: 2^24 < 1.06e9)."""
    rng = np.random.default_rng(23)
    for bits in (4, 6, 8):
        qm = O.QMAX[bits]
        a = rng.integers(-qm, qm + 1, size=(8, 128)).astype(np.int8)
        w = rng.integers(-qm, qm + 1, size=(8, 128)).astype(np.int8)
        want = [[sum(int(a[m, k]) * int(w[n, k]) for k in range(128)) for n in range(8)]
                for m in range(8)]
        assert o.int_gemm_f64(a, w).tolist() == want
    K = 65536
    a = np.full((4, K), 127, np.int8)
    a[1] = -127
    a[2, ::2] = -127
    a[3, :K // 2] = 1  # small terms first, then large ones
    w = np.full((3, K), -127, np.int8)
    w[1] = 127
    w[2, 1::2] = 1

    def exact(m, n):
        # rows and columns are periodic in k with period 2, except row 3,
        # whose halves differ: count the (a, w) value pairs and multiply out
        s = 0
        for half in (0, 1):
            for par in (0, 1):
                k = half * (K // 2) + par
                s += (K // 4) * int(a[m, k]) * int(w[n, k])
        return s

    want = [[exact(m, n) for n in range(3)] for m in range(4)]
    got = o.int_gemm_f64(a, w)
    assert got.tolist() == want
    assert np.abs(got).max() > 2 ** 24


# --------------------------------------------------------------------------- epilogue / bf16

def pin_bf16_rounding_matches_torch(o=O):
    rng = np.random.default_rng(19)
    vals = rng.standard_normal(20000).astype(np.float32) * np.float32(100)
    bits = vals.view(np.uint32).copy()
    bits[:4000] = (bits[:4000] & np.uint32(0xFFFF0000)) | np.uint32(0x8000)  # exact ties
    bits[4000:6000] = (bits[4000:6000] & np.uint32(0xFFFF0000)) | np.uint32(0x7FFF)
    bits[6000:8000] = (bits[6000:8000] & np.uint32(0xFFFF0000)) | np.uint32(0x8001)
    f = bits.view(np.float32)
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(o.f32_to_bf16_bits(f), want)


def pin_epilogue_exact_cases(o=O):
    acc = np.array([[0, 1, -3, 1000], [7, -7, 0, 2048]], dtype=np.int64)
    sa = np.array([0.125, 2.0], dtype=np.float32)
    sw = np.array([0.5, 0.25, 4.0, 2.0 ** -10], dtype=np.float32)
    bias = _bf16([0.0, 1.0, -0.5, 0.25])
    out = o.epilogue(acc, sa, sw, bias)
    want64 = sa[:, None].astype(np.float64) * sw[None, :] * acc + O.bf16_bits_to_f32(bias)[None, :]
    want = torch.from_numpy(want64.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(out, want), "power-of-two scales make every product exact"
    assert np.array_equal(o.epilogue(np.zeros((1, 4), np.int64), sa[:1], sw, bias)[0], bias)


def pin_worked_example(o=O):
    kv = dict(_load_rows("worked_w4_k128.txt")[1:])
    x = np.zeros((1, 128), np.float32)
    x[0, 0] = 8.0
    w = np.zeros((1, 128), np.float32)
    w[0, 0] = 1.0
    r = o.qlinear(_bf16(x), _bf16(w), _bf16([0.25]), 4, 1.0)
    assert int(r["acc"][0, 0]) == int(kv["acc"])
    assert np.all(r["qa"] == int(kv["q_a"])) and np.all(r["qw"] == int(kv["q_w"]))
    assert O.bf16_bits_to_f32(r["out"])[0, 0] == float(kv["out"])


# --------------------------------------------------------------------------- whole layer

def _fp32(v):
    return struct.unpack("f", struct.pack("f", v))[0]


def pin_scalar_loop_tiny(o=O):
    """The whole layer by scalar loops (binary32 emulated by rounding each binary64
    op, which is exact for +,-,*,/ of binary32 operands) against the vectorised oracle."""
    rng = np.random.default_rng(20)
    M, N, K, bits, alpha = 3, 4, 256, 4, 0.9
    x = _bf16(rng.standard_normal((M, K)) * np.where(rng.random(K) < 0.03, 20.0, 1.0))
    w = _bf16(rng.standard_normal((N, K)) * 0.02)
    b = _bf16(rng.standard_normal(N) * 0.01)
    qmax = O.QMAX[bits]

    def quant_row(vals, a, fold):
        v = [float(t) for t in vals]
        for blk in range(K // 128):
            seg = v[blk * 128:(blk + 1) * 128]
            h = 1
            while h < 128:
                for i in range(128):
                    if i & h == 0:
                        p, q_ = seg[i], seg[i + h]
                        seg[i], seg[i + h] = _fp32(p + q_), _fp32(p - q_)
                h *= 2
            v[blk * 128:(blk + 1) * 128] = seg
        amax = max(abs(t) for t in v)
        tt = _fp32(_fp32(a) * amax)
        if tt < 2.0 ** -120:
            return [0] * K, 0.0
        s = _fp32(tt / qmax)
        inv = _fp32(qmax / tt)
        qs = []
        for t in v:
            r = t * inv  # binary64 product of two binary32 values: exact
            qi = round(r)  # Python round is half-to-even
            qs.append(max(-qmax, min(qmax, qi)))
        return qs, _fp32(s * fold)

    xf = O.bf16_bits_to_f32(x)
    wf = O.bf16_bits_to_f32(w)
    bf = O.bf16_bits_to_f32(b)
    QA, SA = zip(*[quant_row(xf[m], alpha, 1.0) for m in range(M)])
    QW, SW = zip(*[quant_row(wf[n], 1.0, 2.0 ** -7) for n in range(N)])
    r = o.qlinear(x, w, b, bits, alpha)
    assert r["qa"].tolist() == [list(t) for t in QA]
    assert r["qw"].tolist() == [list(t) for t in QW]
    assert r["sa"].tolist() == list(SA) and r["sw"].tolist() == list(SW)
    for m in range(M):
        for n in range(N):
            acc = sum(QA[m][k] * QW[n][k] for k in range(K))
            assert r["acc"][m, n] == acc
            y = _fp32(_fp32(_fp32(SA[m] * SW[n]) * float(acc)) + float(bf[n]))
            want = torch.tensor([y], dtype=torch.float32).to(torch.bfloat16).view(torch.int16).item() & 0xFFFF
            assert int(r["out"][m, n]) == want


def pin_folded_vs_literal_normalisation(o=O):
    """Folding 1/sqrt(128) into the weight scale equals the literal normalised rotation."""
    rng = np.random.default_rng(21)
    x = _bf16(rng.standard_normal((48, 512)) * np.where(rng.random(512) < 0.01, 20.0, 1.0))
    w = _bf16(rng.standard_normal((40, 512)) * 0.02)
    bits, alpha = 4, 1.0
    r = o.qlinear(x, w, None, bits, alpha)
    R = O.hadamard_rotation_f64(512)
    qmax = O.QMAX[bits]

    def lit(a, al):
        u = O.bf16_bits_to_f32(a).astype(np.float64) @ R
        s = al * np.abs(u).max(1) / qmax
        return np.clip(np.rint(u / s[:, None]), -qmax, qmax), s

    qa, sa = lit(x, alpha)
    qw, sw = lit(w, 1.0)
    mism = (qa != r["qa"]).mean() + (qw != r["qw"]).mean()
    assert mism <= 1e-3, mism
    y_lit = (qa @ qw.T) * sa[:, None] * sw[None, :]
    y_fold = r["acc"].astype(np.float64) * r["sa"].astype(np.float64)[:, None] * r["sw"].astype(np.float64)[None, :]
    rel = np.linalg.norm(y_lit - y_fold) / np.linalg.norm(y_lit)
    assert rel <= 1e-4, rel


def pin_rotation_improves_sqnr(o=O):
    """Directional check of the pages' claim (rotation spreads outlier channels): on
    inputs with outlier channels the rotated W4A4 layer is closer to the fp64 layer."""
    rng = np.random.default_rng(22)
    K = 1024
    x = _bf16(rng.standard_normal((64, K)) * np.where(rng.random(K) < 0.01, 50.0, 1.0))
    w = _bf16(rng.standard_normal((64, K)) * 0.02)
    ref = O.linear_f64(x, w)

    def sqnr(rot):
        out = O.bf16_bits_to_f32(o.qlinear(x, w, None, 4, 1.0, rotate=rot)["out"]).astype(np.float64)
        return 10 * np.log10((ref ** 2).sum() / ((out - ref) ** 2).sum())

    assert sqnr(True) > sqnr(False) + 1.0


def pin_gelu(o=O):
    v = np.linspace(-6, 6, 2001).astype(np.float32)
    xb = _bf16(v)
    got = O.bf16_bits_to_f32(o.gelu_erf_bf16(xb))
    xt = torch.from_numpy(O.bf16_bits_to_f32(xb).astype(np.float64))
    want = torch.nn.functional.gelu(xt, approximate="none").float().to(torch.bfloat16).float().numpy()
    ulp = np.abs(got - want) / np.maximum(np.abs(want), 1e-30)
    assert np.all((got == want) | (ulp <= 2.0 ** -7))
    # deep negative tail: x*Phi(x) = -phi(x) * (1 - 1/x^2 + 3/x^4 - ...) (Mills ratio
    # asymptotic series), nonzero and accurate to bf16 where 1 + erf cancels.
    xt = np.array([-8.0, -10.0, -12.0], np.float32)
    yt = O.bf16_bits_to_f32(o.gelu_erf_bf16(_bf16(xt))).astype(np.float64)
    x64 = xt.astype(np.float64)
    phi = np.exp(-x64 ** 2 / 2) / math.sqrt(2 * math.pi)
    series = -phi * (1 - 1 / x64 ** 2 + 3 / x64 ** 4 - 15 / x64 ** 6)
    assert np.all(np.abs(yt - series) <= 2.0 ** -7 * np.abs(series))


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_pin(pin):
    pin(O)
