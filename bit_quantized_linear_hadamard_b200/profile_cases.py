"""Small cases of the library's kernels, for profiler captures of one kernel.

    python -m bit_quantized_linear_hadamard_b200.profile_cases CASE [--tokens M]

Each case builds seeded synthetic inputs of the Wan-14B FFN up-projection
shape (K = 5120, N = 13824) with M tokens on cuda:0, runs its kernel three
times through the C ABI and checks the device error word.  The inputs are
sized to exceed the 126 MB L2 at the default M while keeping a few hundred MB
on the device.

Cases:
  sd4_gemm_e4m3   qs_sd4_linear_e4m3 (block-scaled fp8 GEMM, e4m3 x e4m3)
  sd4_gemm_codes  qs_sd4_linear (block-scaled fp8 GEMM decoding SD4 codes)
  sd4_quant_e4m3  qs_sd4_quant_e4m3 (SD4 activation quantiser, e4m3 bytes out)
  gbs_update      qs_gbs_update (normalised L1 change of two layer outputs)
  gelu            qs_gelu_bf16 on an up-projection output (2^24 elements and more:
                  the shared-memory table kernel)
  gemm_w8a8       qs_qlinear, 8-bit activations and weights
  gemm_w4a8       qs_qlinear_mixed, 8-bit activations, 4-bit weights
  gemm_bgr        qs_qlinear_asym, 4-bit activations with code sums, 4-bit weights on
                  bounded (asymmetric) grids
  quant           qs_quant_act at any shape and width (--K, --bits, --alpha, --byte-codes)
  gemm            qs_qlinear_mixed at any shape and widths (--K, --N, --bits-x, --bits-w,
                  --byte-codes: 4-bit activation codes stored one per byte)
"""

from __future__ import annotations

import argparse

import torch

from . import binding as qs

K, N = 5120, 13824


def _inputs(M: int):
    g = torch.Generator(device="cuda").manual_seed(0)
    x = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    w = (torch.randn(N, K, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
    b = (torch.randn(N, device="cuda", generator=g) * 0.01).to(torch.bfloat16)
    return x, w, b


def main(argv=None) -> None:
    p = argparse.ArgumentParser()
    p.add_argument("case", choices=["sd4_gemm_e4m3", "sd4_gemm_e4m3_tiles", "sd4_gemm_codes",
                                    "sd4_quant_e4m3",
                                    "gbs_update", "gelu", "gemm_w8a8", "gemm_w4a8",
                                    "gemm_bgr", "quant", "gemm"])
    p.add_argument("--tokens", type=int, default=None)
    p.add_argument("--K", type=int, default=K)
    p.add_argument("--N", type=int, default=N)
    p.add_argument("--bits", type=int, default=4)
    p.add_argument("--bits-x", type=int, default=4)
    p.add_argument("--bits-w", type=int, default=4)
    p.add_argument("--alpha", type=float, default=1.0)
    p.add_argument("--byte-codes", action="store_true")
    a = p.parse_args(argv)
    qs.load()
    torch.cuda.init()
    if a.case in ("sd4_gemm_e4m3", "sd4_gemm_e4m3_tiles", "sd4_gemm_codes"):
        M = a.tokens or 4096
        x, w, b = _inputs(M)
        cw, mw = qs.sd4_quant(w)
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        if a.case == "sd4_gemm_e4m3":
            x8, mx = qs.sd4_quant_e4m3(x)
            w8 = qs.sd4_decode_e4m3(cw, mw)
            run = lambda: qs.qs_sd4_linear_e4m3(x8, mx, w8, mw, b, M, N, K, out)  # noqa: E731
        elif a.case == "sd4_gemm_e4m3_tiles":
            x8, mx = qs.sd4_quant_e4m3(x)
            w8 = qs.sd4_decode_e4m3(cw, mw)
            xt, wt = qs.sd4_scale_tiles(mx, False), qs.sd4_scale_tiles(mw, True)
            run = lambda: qs.qs_sd4_linear_e4m3_tiles(x8, xt, w8, wt, b, M, N, K, out)  # noqa: E731
        else:
            cx, mx = qs.sd4_quant(x)
            run = lambda: qs.qs_sd4_linear(cx, mx, cw, mw, b, M, N, K, out)  # noqa: E731
    elif a.case == "sd4_quant_e4m3":
        M = a.tokens or 16384
        x, _, _ = _inputs(M)
        x8 = torch.empty((M, K), dtype=torch.uint8, device="cuda")
        mx = torch.empty((M, K // 32), dtype=torch.int16, device="cuda")
        run = lambda: qs.qs_sd4_quant_e4m3(x, M, K, x8, mx)  # noqa: E731
    elif a.case in ("gemm_w8a8", "gemm_w4a8", "gemm_bgr"):
        M = a.tokens or 16384
        x, w, b = _inputs(M)
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        if a.case == "gemm_bgr":
            xp, xs, xr = qs.quant_act_rowsum(x, 4, 1.0)
            wp, ws, wo = qs.pack_weights_bgr(w, 4)
            run = lambda: qs.qs_qlinear_asym(xp, xs, xr, wp, ws, wo, b, M, N, K, 4, out)  # noqa: E731
        else:
            bits_w = 8 if a.case == "gemm_w8a8" else 4
            xp, xs = qs.quant_act(x, 8)
            wp, ws = qs.pack_weights(w, bits_w)
            run = lambda: qs.qlinear(xp, xs, wp, ws, b, 8, K, out=out, bits_w=bits_w)  # noqa: E731
    elif a.case == "quant":
        M = a.tokens or 16384
        g = torch.Generator(device="cuda").manual_seed(0)
        x = torch.randn(M, a.K, device="cuda", generator=g).to(torch.bfloat16)
        flags = qs.QS_FLAG_BYTE_CODES if a.byte_codes else 0
        xp = torch.empty((M, qs.packed_cols(a.K, a.bits, flags)), dtype=torch.uint8,
                         device="cuda")
        xs = torch.empty((M,), dtype=torch.float32, device="cuda")
        run = lambda: qs.qs_quant_act(x, M, a.K, a.bits, a.alpha, flags, xp, xs)  # noqa: E731
    elif a.case == "gemm":
        M = a.tokens or 16384
        g = torch.Generator(device="cuda").manual_seed(0)
        x = torch.randn(M, a.K, device="cuda", generator=g).to(torch.bfloat16)
        w = (torch.randn(a.N, a.K, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
        b = (torch.randn(a.N, device="cuda", generator=g) * 0.01).to(torch.bfloat16)
        flags = qs.QS_FLAG_BYTE_CODES if a.byte_codes else 0
        xp, xs = qs.quant_act(x, a.bits_x, a.alpha, flags)
        wp, ws = qs.pack_weights(w, a.bits_w)
        sx = qs.storage_bits(a.bits_x, flags)
        out = torch.empty((M, a.N), dtype=torch.bfloat16, device="cuda")
        run = lambda: qs.qs_qlinear_mixed(xp, xs, sx, wp, ws, a.bits_w, b, M, a.N, a.K,  # noqa: E731
                                          out)
    elif a.case == "gelu":
        M = a.tokens or 4096
        g = torch.Generator(device="cuda").manual_seed(2)
        y0 = (2.0 * torch.randn(M, N, device="cuda", generator=g)).to(torch.bfloat16)
        y1 = torch.empty_like(y0)
        run = lambda: qs.qs_gelu_bf16(y0, M * N, y1)  # noqa: E731
    else:
        M = a.tokens or 8192
        g = torch.Generator(device="cuda").manual_seed(1)
        y0 = torch.randn(M, N, device="cuda", generator=g).to(torch.bfloat16)
        y1 = (y0.float() + 0.05 * torch.randn(M, N, device="cuda", generator=g)).to(torch.bfloat16)
        state = torch.zeros(qs.QS_GBS_STATE_BYTES, dtype=torch.uint8, device="cuda")
        qs.qs_gbs_reset(state)
        run = lambda: qs.qs_gbs_update(y1, y0, M * N, 0.3, state)  # noqa: E731
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    if qs.qs_device_error() != 0:
        raise SystemExit("a kernel reported a device error")
    print("ok")


if __name__ == "__main__":
    main()
