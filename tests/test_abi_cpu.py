"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, and rejects bad arguments with the documented status before touching
the device."""

import ctypes
import os
import re

import pytest

from bit_quantized_linear_hadamard_b200 import build as qs_build
from bit_quantized_linear_hadamard_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qs.h")

OK, NULL, SHAPE, BITS, ALIGN, RANGE, CUDA, TIMEOUT, PTR = range(9)


@pytest.fixture(scope="module")
def lib():
    qs_build.build()
    return binding.load()


def _declared():
    with open(HEADER) as f:
        src = f.read()
    return sorted(set(re.findall(r"QS_API\s+[\w\s\*]+?\b(qs_\w+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert _declared() == sorted(binding.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings_and_version(lib):
    for code in range(9):
        assert lib.qs_status_str(code)
    assert b"unknown" in lib.qs_status_str(99)
    assert b"sm_100a" in lib.qs_version()


A = ctypes.c_void_p(0x10000)      # 16-byte aligned fake device addresses:
B = ctypes.c_void_p(0x20000)      # validation must reject before any use
C = ctypes.c_void_p(0x30000)
D = ctypes.c_void_p(0x40000)
MIS = ctypes.c_void_p(0x10008)    # 8-byte aligned only
NUL = None


def test_pack_weights_validation(lib):
    f = lib.qs_pack_weights
    assert f(NUL, 256, 512, 4, 0, B, C, NUL) == NULL
    assert f(A, 256, 512, 4, 0, NUL, C, NUL) == NULL
    assert f(A, 256, 512, 4, 0, B, NUL, NUL) == NULL
    assert f(A, 256, 512, 5, 0, B, C, NUL) == BITS
    assert f(A, 256, 500, 4, 0, B, C, NUL) == SHAPE
    assert f(A, 0, 512, 4, 0, B, C, NUL) == SHAPE
    assert f(A, -3, 512, 4, 0, B, C, NUL) == SHAPE
    assert f(A, 256, 0, 4, 0, B, C, NUL) == SHAPE
    assert f(A, 256, 65536 + 128, 4, 0, B, C, NUL) == RANGE
    assert f(A, 256, 512, 4, 4, B, C, NUL) == RANGE          # unknown flag bit
    assert f(MIS, 256, 512, 4, 0, B, C, NUL) == ALIGN


def test_quant_act_validation(lib):
    f = lib.qs_quant_act
    assert f(NUL, 8, 128, 4, 1.0, 0, B, C, NUL) == NULL
    assert f(A, 8, 128, 3, 1.0, 0, B, C, NUL) == BITS
    assert f(A, 8, 130, 4, 1.0, 0, B, C, NUL) == SHAPE
    for alpha in (0.0, -0.5, 1.5, 2.0 ** -15, float("nan"), float("inf")):
        assert f(A, 8, 128, 4, alpha, 0, B, C, NUL) == RANGE, alpha
    assert f(A, 8, 128, 8, 1.0, 0x10, B, C, NUL) == RANGE
    assert f(A, 8, 128, 8, 1.0, 0, MIS, C, NUL) == ALIGN
    assert f(A, 8, 128, 8, 1.0, 0, B, ctypes.c_void_p(0x30004), NUL) == ALIGN


def test_qlinear_validation(lib):
    f = lib.qs_qlinear
    assert f(NUL, B, C, D, NUL, 8, 256, 128, 4, A, NUL) == NULL
    assert f(A, NUL, C, D, NUL, 8, 256, 128, 4, B, NUL) == NULL
    assert f(A, B, C, NUL, NUL, 8, 256, 128, 4, B, NUL) == NULL
    assert f(A, B, C, D, NUL, 8, 256, 128, 4, NUL, NUL) == NULL
    assert f(A, B, C, D, NUL, 8, 264, 128, 4, A, NUL) == SHAPE   # N % 16
    assert f(A, B, C, D, NUL, 8, 256, 192, 4, A, NUL) == SHAPE   # K % 128
    assert f(A, B, C, D, NUL, 0, 256, 128, 4, A, NUL) == SHAPE
    assert f(A, B, C, D, NUL, 8, 256, 128, 5, A, NUL) == BITS
    assert f(A, B, C, D, NUL, 8, 256, 128, 16, A, NUL) == BITS
    assert f(A, B, C, D, NUL, 8, 256, 2 * 65536, 8, A, NUL) == RANGE
    assert f(A, B, C, D, MIS, 8, 256, 128, 4, A, NUL) == ALIGN   # bias
    assert f(MIS, B, C, D, NUL, 8, 256, 128, 4, A, NUL) == ALIGN


def test_mixed_validation(lib):
    f = lib.qs_qlinear_mixed
    assert f(NUL, B, 8, C, D, 4, NUL, 8, 256, 128, A, NUL) == NULL
    assert f(A, B, 8, C, NUL, 4, NUL, 8, 256, 128, A, NUL) == NULL
    assert f(A, B, 7, C, D, 4, NUL, 8, 256, 128, A, NUL) == BITS
    assert f(A, B, 8, C, D, 2, NUL, 8, 256, 128, A, NUL) == BITS
    assert f(A, B, 8, C, D, 4, NUL, 8, 264, 128, A, NUL) == SHAPE
    assert f(A, B, 6, C, D, 4, MIS, 8, 256, 128, A, NUL) == ALIGN
    g = lib.qs_qgemm_s32_mixed
    assert g(A, 8, NUL, 4, 8, 256, 128, C, NUL) == NULL
    assert g(A, 8, B, 3, 8, 256, 128, C, NUL) == BITS
    assert g(A, 6, B, 4, 8, 256, 192, C, NUL) == SHAPE
    h = lib.qs_linear_mixed
    need = lib.qs_linear_workspace_bytes(8, 128, 8)
    assert h(A, 8, 128, 1.0, 8, B, C, 4, NUL, 256, D, need, A, NUL) == PTR  # fake addresses
    assert h(A, 8, 128, 1.0, 8, B, C, 4, NUL, 256, D, need - 1, A, NUL) == RANGE
    assert h(A, 8, 128, 1.0, 9, B, C, 4, NUL, 256, D, need, A, NUL) == BITS
    assert h(A, 8, 128, 0.0, 8, B, C, 4, NUL, 256, D, need, A, NUL) == RANGE


def test_qgemm_and_gelu_validation(lib):
    assert lib.qs_qgemm_s32(NUL, B, 8, 256, 128, 4, C, NUL) == NULL
    assert lib.qs_qgemm_s32(A, B, 8, 250, 128, 4, C, NUL) == SHAPE
    assert lib.qs_qgemm_s32(A, B, 8, 256, 128, 2, C, NUL) == BITS
    assert lib.qs_qgemm_s32(A, B, 8, 256, 128, 4, MIS, NUL) == ALIGN
    assert lib.qs_gelu_bf16(NUL, 16, B, NUL) == NULL
    assert lib.qs_gelu_bf16(A, 0, B, NUL) == SHAPE
    assert lib.qs_gelu_bf16(A, 16, MIS, NUL) == ALIGN


def test_host_memory_is_rejected(lib):
    # Well-formed arguments pointing at host memory: rejected as QS_ERR_PTR (on a
    # machine without a GPU the pointer query fails the same way).
    buf = ctypes.create_string_buffer(4096 + 16)
    base = (ctypes.addressof(buf) + 15) // 16 * 16
    p = ctypes.c_void_p(base)
    st = lib.qs_quant_act(p, 1, 128, 4, 1.0, 0, ctypes.c_void_p(base + 1024),
                          ctypes.c_void_p(base + 2048), NUL)
    assert st == PTR


def test_binding_raises_without_cuda_tensors():
    import torch
    with pytest.raises(TypeError):
        binding.quant_act(torch.zeros(4, 128, dtype=torch.bfloat16), 4)


def test_quant_linear_rejects_an_unknown_code_layout():
    import torch
    with pytest.raises(ValueError):
        binding.QuantLinear(torch.zeros((16, 128), dtype=torch.bfloat16), None, 4,
                            act_codes="nibbles")


def test_storage_widths():
    assert binding.storage_bits(4) == 4
    assert binding.storage_bits(4, binding.QS_FLAG_BYTE_CODES) == 8
    assert binding.storage_bits(8) == 8
    assert binding.packed_cols(5120, 4) == 2560
    assert binding.packed_cols(5120, 4, binding.QS_FLAG_BYTE_CODES) == 5120
    assert binding.packed_cols(5120, 6) == 5120 and binding.packed_cols(5120, 8) == 5120


def test_linear_validation_and_workspace(lib):
    assert lib.qs_linear_workspace_bytes(256, 512, 4) == 256 * 256 + 4 * 256
    assert lib.qs_linear_workspace_bytes(3, 128, 4) == 256 + 12          # packed part rounded to 256
    assert lib.qs_linear_workspace_bytes(3, 128, 8) == 512 + 12
    assert lib.qs_linear_workspace_bytes(3, 128, 6) == 512 + 12          # 6-bit codes take a byte
    assert lib.qs_linear_workspace_bytes(3, 100, 4) == -1
    assert lib.qs_linear_workspace_bytes(3, 128, 5) == -1
    need = lib.qs_linear_workspace_bytes(8, 128, 4)
    f = lib.qs_linear
    assert f(NUL, 8, 128, 1.0, B, C, NUL, 256, 4, D, need, A, NUL) == NULL
    assert f(A, 8, 128, 1.0, B, C, NUL, 256, 4, NUL, need, D, NUL) == NULL
    assert f(A, 8, 128, 1.0, B, C, NUL, 250, 4, D, need, A, NUL) == SHAPE
    assert f(A, 8, 128, 1.5, B, C, NUL, 256, 4, D, need, A, NUL) == RANGE
    assert f(A, 8, 128, 1.0, B, C, NUL, 256, 4, D, need - 1, A, NUL) == RANGE
    assert f(MIS, 8, 128, 1.0, B, C, NUL, 256, 4, D, need, A, NUL) == ALIGN
    assert f(A, 8, 128, 1.0, B, C, MIS, 256, 4, D, need, A, NUL) == ALIGN


def test_selftest_timeout_validation(lib):
    assert lib.qs_selftest_timeout(0, NUL) == RANGE
    assert lib.qs_selftest_timeout(1000001, NUL) == RANGE


def test_gbs_validation(lib):
    assert lib.qs_gbs_reset(NUL, NUL) == NULL
    assert lib.qs_gbs_reset(MIS, NUL) == ALIGN
    up = lib.qs_gbs_update
    assert up(NUL, B, 64, 0.5, C, NUL) == NULL
    assert up(A, B, 64, 0.5, NUL, NUL) == NULL
    assert up(A, B, 0, 0.5, C, NUL) == SHAPE
    for delta in (-0.5, float("nan"), float("inf")):
        assert up(A, B, 64, delta, C, NUL) == RANGE, delta
    assert up(A, MIS, 64, 0.5, C, NUL) == ALIGN
    assert up(A, B, 64, 0.5, ctypes.c_void_p(0x30008), NUL) == ALIGN
    f = lib.qs_linear_gbs
    need = lib.qs_linear_workspace_bytes(8, 128, 8)
    args = [A, 8, 128, 1.0, B, C, B, C, NUL, 256, D, A, need, A, NUL]
    bad = list(args); bad[6] = NUL
    assert f(*bad) == NULL                                  # no 8-bit weights
    bad = list(args); bad[9] = 250
    assert f(*bad) == SHAPE
    bad = list(args); bad[12] = need - 1
    assert f(*bad) == RANGE                                 # workspace sized for 8 bits
    bad = list(args); bad[10] = ctypes.c_void_p(0x40008)
    assert f(*bad) == ALIGN                                 # state
    assert f(*args) == PTR                                  # fake addresses


def test_gbs_state_layout_matches_the_header(tmp_path):
    """sizeof and offsets of qs_gbs_state as a C compiler lays it out."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stddef.h>\n#include <stdio.h>\n#include "qs.h"\n'
        'int main(void) { printf("%zu %zu %zu %zu %zu %zu\\n", sizeof(qs_gbs_state), '
        'offsetof(qs_gbs_state, acc), offsetof(qs_gbs_state, last_d), '
        'offsetof(qs_gbs_state, bits), offsetof(qs_gbs_state, step), '
        'offsetof(qs_gbs_state, partial)); return 0; }\n')
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    assert [int(v) for v in out] == [binding.QS_GBS_STATE_BYTES, 0, 8, 16, 20, 32]


def test_bgr_validation(lib):
    f = lib.qs_pack_weights_bgr
    assert f(NUL, 16, 128, 4, 0, 64, 8, B, C, D, NUL) == NULL
    assert f(A, 16, 128, 4, 0, 64, 8, B, C, NUL, NUL) == NULL
    assert f(A, 16, 128, 6, 0, 64, 8, B, C, D, NUL) == BITS      # BGR grids: 4 or 8 bits
    assert f(A, 16, 130, 4, 0, 64, 8, B, C, D, NUL) == SHAPE
    assert f(A, 16, 32768 + 128, 4, 0, 64, 8, B, C, D, NUL) == RANGE  # row held on chip
    for cand, iters in ((0, 8), (257, 8), (64, -1), (64, 65)):
        assert f(A, 16, 128, 4, 0, cand, iters, B, C, D, NUL) == RANGE, (cand, iters)
    assert f(A, 16, 128, 4, 0, 64, 8, B, C, ctypes.c_void_p(0x40004), NUL) == ALIGN
    g = lib.qs_quant_act_rowsum
    assert g(A, 8, 128, 4, 1.0, 0, B, C, NUL, NUL) == NULL
    assert g(A, 8, 128, 4, 1.0, 0, B, C, ctypes.c_void_p(0x40004), NUL) == ALIGN
    assert g(A, 8, 128, 5, 1.0, 0, B, C, D, NUL) == BITS
    h = lib.qs_qlinear_asym
    assert h(A, B, C, D, A, B, NUL, 8, 256, 128, 6, C, NUL) == BITS
    assert h(A, B, NUL, D, A, B, NUL, 8, 256, 128, 4, C, NUL) == NULL
    assert h(A, B, C, D, A, B, NUL, 8, 264, 128, 4, C, NUL) == SHAPE
    assert lib.qs_qgemm_s32_asym(A, B, C, NUL, 8, 256, 128, 4, D, NUL) == NULL
    assert lib.qs_linear_bgr_workspace_bytes(3, 128, 4) == 256 + 256 + 12
    assert lib.qs_linear_bgr_workspace_bytes(3, 128, 6) == -1
    need = lib.qs_linear_bgr_workspace_bytes(8, 128, 4)
    k = lib.qs_linear_bgr
    assert k(A, 8, 128, 1.0, B, C, D, NUL, 256, 4, A, need - 1, B, NUL) == RANGE
    assert k(A, 8, 128, 1.0, B, C, NUL, NUL, 256, 4, A, need, B, NUL) == NULL


def test_sd4_validation(lib):
    q = lib.qs_sd4_quant
    assert q(NUL, 8, 256, B, C, NUL) == NULL
    assert q(A, 8, 384, B, C, NUL) == SHAPE                 # K % 256
    assert q(A, 8, 256, B, ctypes.c_void_p(0x30008), NUL) == ALIGN
    f = lib.qs_sd4_linear
    assert f(A, B, C, NUL, NUL, 8, 256, 256, D, NUL) == NULL
    assert f(A, B, C, D, NUL, 8, 264, 256, D, NUL) == SHAPE  # N % 16
    assert f(A, B, C, D, NUL, 8, 256, 65536 + 256, D, NUL) == RANGE
    assert lib.qs_sd4_decode(A, B, 4, 128, C, NUL) == SHAPE
    assert lib.qs_sd4_linear_wdec(A, B, NUL, NUL, 8, 256, 256, D, NUL) == NULL
    g = lib.qs_sd4_quant_decomp
    assert g(A, 8, 256, NUL, 4, C, D, NUL) == NULL          # rows
    assert g(A, 8, 256, B, 0, C, D, NUL) == SHAPE           # no salient rows
    assert g(A, 0, 256, B, 4, C, D, NUL) == SHAPE
    assert g(A, 8, 32768 + 256, B, 4, C, D, NUL) == RANGE   # 2K codes per row
    assert g(A, 8, 256, ctypes.c_void_p(0x20002), 4, C, D, NUL) == ALIGN
    h = lib.qs_sd4_linear_decomp
    assert h(A, B, C, 4, NUL, D, NUL, NUL, 8, 256, 256, D, NUL) == NULL     # no weights
    assert h(A, B, C, 4, A, NUL, NUL, NUL, 8, 256, 256, D, NUL) == NULL     # codes without words
    assert h(A, B, C, 4, NUL, NUL, D, NUL, 8, 256, 256, D, NUL) == NULL     # e4m3 without words
    assert h(A, B, C, 4, NUL, D, D, NUL, 8, 264, 256, D, NUL) == SHAPE
    assert h(A, B, C, 4, NUL, D, D, NUL, 8, 256, 384, D, NUL) == SHAPE
    assert h(A, B, C, 4, NUL, D, D, NUL, 8, 256, 32768 + 256, D, NUL) == RANGE
    assert h(A, B, C, 4, NUL, D, MIS, NUL, 8, 256, 256, D, NUL) == ALIGN
    assert h(A, B, ctypes.c_void_p(0x30002), 4, A, B, NUL, NUL, 8, 256, 256, D, NUL) == ALIGN
    assert lib.qs_sd4_decode_e4m3(A, B, 4, 128, C, NUL) == SHAPE
    assert lib.qs_sd4_decode_e4m3(A, NUL, 4, 256, C, NUL) == NULL
    assert lib.qs_sd4_decode_e4m3(A, B, 4, 256, MIS, NUL) == ALIGN
    e = lib.qs_sd4_linear_e4m3w
    assert e(A, B, C, NUL, NUL, 8, 256, 256, D, NUL) == NULL                # block words required
    assert e(A, B, C, D, NUL, 8, 200, 256, D, NUL) == SHAPE
    assert e(A, B, C, D, NUL, 8, 256, 256 + 128, D, NUL) == SHAPE
    assert e(A, B, C, D, MIS, 8, 256, 256, D, NUL) == ALIGN
    assert lib.qs_sd4_quant_e4m3(A, 8, 384, B, C, NUL) == SHAPE
    assert lib.qs_sd4_quant_e4m3(A, 8, 256, NUL, C, NUL) == NULL
    f8 = lib.qs_sd4_linear_e4m3
    assert f8(A, B, C, NUL, NUL, 8, 256, 256, D, NUL) == NULL
    assert f8(A, B, C, D, NUL, 8, 248, 256, D, NUL) == SHAPE
    assert f8(MIS, B, C, D, NUL, 8, 256, 256, D, NUL) == ALIGN


def test_sd4_scale_tiles_sizes_and_validation(lib):
    nb = lib.qs_sd4_scale_tiles_bytes
    # activations: groups of 128 rows, 512 bytes per group and 128-element K step
    assert nb(128, 256, 0) == 1 * 2 * 512
    assert nb(129, 256, 0) == 2 * 2 * 512
    assert nb(32760, 5120, 0) == 256 * 40 * 512
    # weights: groups of 192 rows in whole pairs (one 384-column GEMM tile), 1024 bytes
    assert nb(16, 256, 1) == 2 * 2 * 1024
    assert nb(384, 256, 1) == 2 * 2 * 1024
    assert nb(385, 256, 1) == 4 * 2 * 1024
    assert nb(13824, 5120, 1) == 72 * 40 * 1024
    assert nb(0, 256, 0) == -1 and nb(8, 384, 0) == -1 and nb(8, 256 + 65536, 1) == -1
    t = lib.qs_sd4_scale_tiles
    need = nb(8, 256, 0)
    assert t(NUL, 8, 256, 0, B, need, NUL) == NULL
    assert t(A, 8, 384, 0, B, need, NUL) == SHAPE
    assert t(A, 8, 256, 2, B, need, NUL) == RANGE
    assert t(A, 8, 256, 0, B, need - 16, NUL) == RANGE      # buffer too small
    assert t(MIS, 8, 256, 0, B, need, NUL) == ALIGN
    g = lib.qs_sd4_linear_e4m3_tiles
    assert g(A, NUL, C, D, NUL, 8, 256, 256, D, NUL) == NULL
    assert g(A, B, C, D, NUL, 8, 248, 256, D, NUL) == SHAPE
    assert g(A, B, C, D, NUL, 8, 256, 384, D, NUL) == SHAPE
    assert g(A, B, C, D, NUL, 8, 256, 65536 + 256, D, NUL) == RANGE
    assert g(A, MIS, C, D, NUL, 8, 256, 256, D, NUL) == ALIGN
