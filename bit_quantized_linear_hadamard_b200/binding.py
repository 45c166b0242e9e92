"""ctypes binding of libqs.so.

The functions named like the C entry points (``qs_pack_weights``,
``qs_quant_act``, ``qs_qlinear``, ``qs_qlinear_mixed``, ``qs_qgemm_s32``,
``qs_gelu_bf16``, ...) take torch
CUDA tensors and only marshal their pointers, sizes and the stream into the C
call; every step of the computation runs in the library's kernels.  The
lower-case helpers (``pack_weights``, ``quant_act``, ``qlinear``, ...) allocate
the output tensors with torch and call those.

There is no fallback: if libqs.so has not been built, or a call returns an
error status, a ``QSError`` is raised.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqs.so")

QS_FLAG_NO_ROTATE = 1
QS_FLAG_BYTE_CODES = 2
QS_MAX_K = 65536
STATUS = {0: "QS_OK", 1: "QS_ERR_NULL", 2: "QS_ERR_SHAPE", 3: "QS_ERR_BITS", 4: "QS_ERR_ALIGN",
          5: "QS_ERR_RANGE", 6: "QS_ERR_CUDA", 7: "QS_ERR_TIMEOUT", 8: "QS_ERR_PTR"}
EXPORTS = ("qs_pack_weights", "qs_quant_act", "qs_qlinear", "qs_qlinear_mixed", "qs_qgemm_s32",
           "qs_qgemm_s32_mixed", "qs_gelu_bf16", "qs_linear_workspace_bytes", "qs_linear",
           "qs_linear_mixed", "qs_linear_ex", "qs_linear_noalloc", "qs_pack_weights_bgr",
           "qs_quant_act_rowsum", "qs_qlinear_asym", "qs_qgemm_s32_asym",
           "qs_linear_bgr_workspace_bytes", "qs_linear_bgr", "qs_sd4_quant", "qs_sd4_quant_e4m3",
           "qs_sd4_linear", "qs_sd4_decode", "qs_sd4_linear_wdec", "qs_sd4_decode_e4m3",
           "qs_sd4_linear_e4m3w", "qs_sd4_linear_e4m3", "qs_sd4_scale_tiles_bytes",
           "qs_sd4_scale_tiles", "qs_sd4_linear_e4m3_tiles", "qs_sd4_quant_decomp",
           "qs_sd4_linear_decomp", "qs_gbs_reset", "qs_gbs_update", "qs_linear_gbs",
           "qs_selftest_timeout", "qs_device_error", "qs_status_str", "qs_version")
BITS = (4, 6, 8)
QS_GBS_MAX_BLOCKS = 1024
# sizeof(qs_gbs_state): acc, last_d (f64), bits, step, blocks_done, reserved (i32), partials
QS_GBS_STATE_BYTES = 8 + 8 + 4 * 4 + 2 * QS_GBS_MAX_BLOCKS * 8
QS_NOALLOC_SCRATCH_BYTES = 8 << 20


class QSError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({_status_str(status)})")


_lib = None


def load() -> ctypes.CDLL:
    """Loads libqs.so (once) and declares the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is not built; run `python -m bit_quantized_linear_hadamard_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, u32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint, ctypes.c_float
    L.qs_pack_weights.argtypes = [vp, i64, i64, i32, u32, vp, vp, vp]
    L.qs_quant_act.argtypes = [vp, i64, i64, i32, f32, u32, vp, vp, vp]
    L.qs_qlinear.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, vp, vp]
    L.qs_qlinear_mixed.argtypes = [vp, vp, i32, vp, vp, i32, vp, i64, i64, i64, vp, vp]
    L.qs_qgemm_s32.argtypes = [vp, vp, i64, i64, i64, i32, vp, vp]
    L.qs_qgemm_s32_mixed.argtypes = [vp, i32, vp, i32, i64, i64, i64, vp, vp]
    L.qs_gelu_bf16.argtypes = [vp, i64, vp, vp]
    L.qs_linear_workspace_bytes.argtypes = [i64, i64, i32]
    L.qs_linear_workspace_bytes.restype = i64
    L.qs_linear.argtypes = [vp, i64, i64, f32, vp, vp, vp, i64, i32, vp, i64, vp, vp]
    L.qs_linear_mixed.argtypes = [vp, i64, i64, f32, i32, vp, vp, i32, vp, i64, vp, i64, vp, vp]
    L.qs_linear_ex.argtypes = [vp, i64, i64, f32, i32, u32, vp, vp, i32, vp, i64, vp, i64, vp, vp]
    L.qs_linear_noalloc.argtypes = [vp, i64, i64, f32, vp, vp, vp, i64, i32, vp, vp]
    f64 = ctypes.c_double
    L.qs_pack_weights_bgr.argtypes = [vp, i64, i64, i32, u32, i32, i32, vp, vp, vp, vp]
    L.qs_quant_act_rowsum.argtypes = [vp, i64, i64, i32, f32, u32, vp, vp, vp, vp]
    L.qs_qlinear_asym.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, vp, vp]
    L.qs_qgemm_s32_asym.argtypes = [vp, vp, vp, vp, i64, i64, i64, i32, vp, vp]
    L.qs_linear_bgr_workspace_bytes.argtypes = [i64, i64, i32]
    L.qs_linear_bgr_workspace_bytes.restype = i64
    L.qs_linear_bgr.argtypes = [vp, i64, i64, f32, vp, vp, vp, vp, i64, i32, vp, i64, vp, vp]
    L.qs_sd4_quant.argtypes = [vp, i64, i64, vp, vp, vp]
    L.qs_sd4_linear.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp, vp]
    L.qs_sd4_decode.argtypes = [vp, vp, i64, i64, vp, vp]
    L.qs_sd4_linear_wdec.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, vp]
    L.qs_sd4_quant_decomp.argtypes = [vp, i64, i64, vp, i64, vp, vp, vp]
    L.qs_sd4_linear_decomp.argtypes = [vp, vp, vp, i64, vp, vp, vp, vp, i64, i64, i64, vp, vp]
    L.qs_sd4_decode_e4m3.argtypes = [vp, vp, i64, i64, vp, vp]
    L.qs_sd4_linear_e4m3w.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp, vp]
    L.qs_sd4_quant_e4m3.argtypes = [vp, i64, i64, vp, vp, vp]
    L.qs_sd4_linear_e4m3.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp, vp]
    L.qs_sd4_scale_tiles_bytes.argtypes = [i64, i64, i32]
    L.qs_sd4_scale_tiles_bytes.restype = i64
    L.qs_sd4_scale_tiles.argtypes = [vp, i64, i64, i32, vp, i64, vp]
    L.qs_sd4_linear_e4m3_tiles.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp, vp]
    L.qs_gbs_reset.argtypes = [vp, vp]
    L.qs_gbs_update.argtypes = [vp, vp, i64, f64, vp, vp]
    L.qs_linear_gbs.argtypes = [vp, i64, i64, f32, vp, vp, vp, vp, vp, i64, vp, vp, i64, vp, vp]
    L.qs_selftest_timeout.argtypes = [i64, vp]
    L.qs_device_error.argtypes = [vp]
    L.qs_status_str.argtypes = [i32]
    L.qs_status_str.restype = ctypes.c_char_p
    L.qs_version.restype = ctypes.c_char_p
    for name in ("qs_pack_weights", "qs_quant_act", "qs_qlinear", "qs_qlinear_mixed",
                 "qs_qgemm_s32", "qs_qgemm_s32_mixed", "qs_gelu_bf16", "qs_linear",
                 "qs_linear_mixed", "qs_linear_ex", "qs_linear_noalloc", "qs_pack_weights_bgr",
                 "qs_quant_act_rowsum", "qs_qlinear_asym", "qs_qgemm_s32_asym", "qs_linear_bgr",
                 "qs_sd4_quant", "qs_sd4_quant_e4m3", "qs_sd4_linear", "qs_sd4_decode",
                 "qs_sd4_linear_wdec", "qs_sd4_decode_e4m3", "qs_sd4_linear_e4m3w",
                 "qs_sd4_linear_e4m3", "qs_sd4_scale_tiles", "qs_sd4_linear_e4m3_tiles",
                 "qs_sd4_quant_decomp", "qs_sd4_linear_decomp",
                 "qs_gbs_reset", "qs_gbs_update", "qs_linear_gbs", "qs_selftest_timeout",
                 "qs_device_error"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def _status_str(status: int) -> str:
    try:
        return load().qs_status_str(status).decode()
    except Exception:  # noqa: BLE001 - only used to decorate an error message
        return "?"


def _check(status: int, where: str) -> None:
    if status != 0:
        raise QSError(status, where)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _cuda(t, dtype, name):
    if t is None:
        return
    if not (isinstance(t, torch.Tensor) and t.is_cuda):
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# --------------------------------------------------------------------------- C mirrors

def qs_pack_weights(w, N, K, bits, flags, w_packed, w_scale, stream=None):
    _cuda(w, torch.bfloat16, "w")
    _cuda(w_packed, torch.uint8, "w_packed")
    _cuda(w_scale, torch.float32, "w_scale")
    _check(load().qs_pack_weights(_p(w), N, K, bits, flags, _p(w_packed), _p(w_scale), _s(stream)),
           "qs_pack_weights")


def qs_quant_act(x, M, K, bits, alpha, flags, x_packed, x_scale, stream=None):
    _cuda(x, torch.bfloat16, "x")
    _cuda(x_packed, torch.uint8, "x_packed")
    _cuda(x_scale, torch.float32, "x_scale")
    _check(load().qs_quant_act(_p(x), M, K, bits, float(alpha), flags, _p(x_packed), _p(x_scale),
                               _s(stream)), "qs_quant_act")


def qs_qlinear(x_packed, x_scale, w_packed, w_scale, bias, M, N, K, bits, out, stream=None):
    _cuda(x_packed, torch.uint8, "x_packed")
    _cuda(w_packed, torch.uint8, "w_packed")
    _cuda(x_scale, torch.float32, "x_scale")
    _cuda(w_scale, torch.float32, "w_scale")
    _cuda(bias, torch.bfloat16, "bias")
    _cuda(out, torch.bfloat16, "out")
    _check(load().qs_qlinear(_p(x_packed), _p(x_scale), _p(w_packed), _p(w_scale), _p(bias),
                             M, N, K, bits, _p(out), _s(stream)), "qs_qlinear")


def qs_qlinear_mixed(x_packed, x_scale, bits_x, w_packed, w_scale, bits_w, bias, M, N, K, out,
                     stream=None):
    _cuda(x_packed, torch.uint8, "x_packed")
    _cuda(w_packed, torch.uint8, "w_packed")
    _cuda(x_scale, torch.float32, "x_scale")
    _cuda(w_scale, torch.float32, "w_scale")
    _cuda(bias, torch.bfloat16, "bias")
    _cuda(out, torch.bfloat16, "out")
    _check(load().qs_qlinear_mixed(_p(x_packed), _p(x_scale), bits_x, _p(w_packed), _p(w_scale),
                                   bits_w, _p(bias), M, N, K, _p(out), _s(stream)),
           "qs_qlinear_mixed")


def qs_qgemm_s32_mixed(x_packed, bits_x, w_packed, bits_w, M, N, K, acc, stream=None):
    _cuda(x_packed, torch.uint8, "x_packed")
    _cuda(w_packed, torch.uint8, "w_packed")
    _cuda(acc, torch.int32, "acc")
    _check(load().qs_qgemm_s32_mixed(_p(x_packed), bits_x, _p(w_packed), bits_w, M, N, K, _p(acc),
                                     _s(stream)), "qs_qgemm_s32_mixed")


def qs_qgemm_s32(x_packed, w_packed, M, N, K, bits, acc, stream=None):
    _cuda(x_packed, torch.uint8, "x_packed")
    _cuda(w_packed, torch.uint8, "w_packed")
    _cuda(acc, torch.int32, "acc")
    _check(load().qs_qgemm_s32(_p(x_packed), _p(w_packed), M, N, K, bits, _p(acc), _s(stream)),
           "qs_qgemm_s32")


def qs_gelu_bf16(x, n, y, stream=None):
    _cuda(x, torch.bfloat16, "x")
    _cuda(y, torch.bfloat16, "y")
    _check(load().qs_gelu_bf16(_p(x), n, _p(y), _s(stream)), "qs_gelu_bf16")


def qs_linear_workspace_bytes(M, K, bits) -> int:
    return int(load().qs_linear_workspace_bytes(M, K, bits))


def qs_linear(x, M, K, alpha, w_packed, w_scale, bias, N, bits, workspace, workspace_bytes, out,
              stream=None):
    _cuda(x, torch.bfloat16, "x")
    _cuda(w_packed, torch.uint8, "w_packed")
    _cuda(w_scale, torch.float32, "w_scale")
    _cuda(bias, torch.bfloat16, "bias")
    _cuda(workspace, torch.uint8, "workspace")
    _cuda(out, torch.bfloat16, "out")
    _check(load().qs_linear(_p(x), M, K, float(alpha), _p(w_packed), _p(w_scale), _p(bias), N, bits,
                            _p(workspace), workspace_bytes, _p(out), _s(stream)), "qs_linear")


def qs_linear_mixed(x, M, K, alpha, bits_x, w_packed, w_scale, bits_w, bias, N, workspace,
                    workspace_bytes, out, stream=None):
    _cuda(x, torch.bfloat16, "x")
    _cuda(w_packed, torch.uint8, "w_packed")
    _cuda(w_scale, torch.float32, "w_scale")
    _cuda(bias, torch.bfloat16, "bias")
    _cuda(workspace, torch.uint8, "workspace")
    _cuda(out, torch.bfloat16, "out")
    _check(load().qs_linear_mixed(_p(x), M, K, float(alpha), bits_x, _p(w_packed), _p(w_scale),
                                  bits_w, _p(bias), N, _p(workspace), workspace_bytes, _p(out),
                                  _s(stream)), "qs_linear_mixed")


def qs_linear_ex(x, M, K, alpha, bits_x, x_flags, w_packed, w_scale, bits_w, bias, N, workspace,
                 workspace_bytes, out, stream=None):
    _cuda(x, torch.bfloat16, "x")
    _cuda(w_packed, torch.uint8, "w_packed")
    _cuda(w_scale, torch.float32, "w_scale")
    _cuda(bias, torch.bfloat16, "bias")
    _cuda(workspace, torch.uint8, "workspace")
    _cuda(out, torch.bfloat16, "out")
    _check(load().qs_linear_ex(_p(x), M, K, float(alpha), bits_x, x_flags, _p(w_packed),
                               _p(w_scale), bits_w, _p(bias), N, _p(workspace), workspace_bytes,
                               _p(out), _s(stream)), "qs_linear_ex")


def qs_linear_noalloc(x, M, K, alpha, w_packed, w_scale, bias, N, bits, out, stream=None):
    """qs_linear on the library's own fixed scratch buffer (for callers that
    cannot allocate device memory when they run the layer); nothing is allocated."""
    _cuda(x, torch.bfloat16, "x")
    _cuda(w_packed, torch.uint8, "w_packed")
    _cuda(w_scale, torch.float32, "w_scale")
    _cuda(bias, torch.bfloat16, "bias")
    _cuda(out, torch.bfloat16, "out")
    _check(load().qs_linear_noalloc(_p(x), M, K, float(alpha), _p(w_packed), _p(w_scale), _p(bias),
                                    N, bits, _p(out), _s(stream)), "qs_linear_noalloc")


def qs_pack_weights_bgr(w, N, K, bits, flags, candidates, iterations, w_packed, w_scale,
                        w_offset, stream=None):
    _cuda(w, torch.bfloat16, "w")
    _cuda(w_packed, torch.uint8, "w_packed")
    _cuda(w_scale, torch.float32, "w_scale")
    _cuda(w_offset, torch.int32, "w_offset")
    _check(load().qs_pack_weights_bgr(_p(w), N, K, bits, flags, candidates, iterations,
                                      _p(w_packed), _p(w_scale), _p(w_offset), _s(stream)),
           "qs_pack_weights_bgr")


def qs_quant_act_rowsum(x, M, K, bits, alpha, flags, x_packed, x_scale, x_rowsum, stream=None):
    _cuda(x, torch.bfloat16, "x")
    _cuda(x_packed, torch.uint8, "x_packed")
    _cuda(x_scale, torch.float32, "x_scale")
    _cuda(x_rowsum, torch.int32, "x_rowsum")
    _check(load().qs_quant_act_rowsum(_p(x), M, K, bits, float(alpha), flags, _p(x_packed),
                                      _p(x_scale), _p(x_rowsum), _s(stream)),
           "qs_quant_act_rowsum")


def qs_qlinear_asym(x_packed, x_scale, x_rowsum, w_packed, w_scale, w_offset, bias, M, N, K,
                    bits, out, stream=None):
    for t, name, dt in ((x_packed, "x_packed", torch.uint8), (w_packed, "w_packed", torch.uint8),
                        (x_scale, "x_scale", torch.float32), (w_scale, "w_scale", torch.float32),
                        (x_rowsum, "x_rowsum", torch.int32), (w_offset, "w_offset", torch.int32),
                        (bias, "bias", torch.bfloat16), (out, "out", torch.bfloat16)):
        _cuda(t, dt, name)
    _check(load().qs_qlinear_asym(_p(x_packed), _p(x_scale), _p(x_rowsum), _p(w_packed),
                                  _p(w_scale), _p(w_offset), _p(bias), M, N, K, bits, _p(out),
                                  _s(stream)), "qs_qlinear_asym")


def qs_qgemm_s32_asym(x_packed, x_rowsum, w_packed, w_offset, M, N, K, bits, acc, stream=None):
    for t, name, dt in ((x_packed, "x_packed", torch.uint8), (w_packed, "w_packed", torch.uint8),
                        (x_rowsum, "x_rowsum", torch.int32), (w_offset, "w_offset", torch.int32),
                        (acc, "acc", torch.int32)):
        _cuda(t, dt, name)
    _check(load().qs_qgemm_s32_asym(_p(x_packed), _p(x_rowsum), _p(w_packed), _p(w_offset), M, N,
                                    K, bits, _p(acc), _s(stream)), "qs_qgemm_s32_asym")


def qs_linear_bgr_workspace_bytes(M, K, bits) -> int:
    return int(load().qs_linear_bgr_workspace_bytes(M, K, bits))


def qs_linear_bgr(x, M, K, alpha, w_packed, w_scale, w_offset, bias, N, bits, workspace,
                  workspace_bytes, out, stream=None):
    for t, name, dt in ((x, "x", torch.bfloat16), (w_packed, "w_packed", torch.uint8),
                        (w_scale, "w_scale", torch.float32), (w_offset, "w_offset", torch.int32),
                        (bias, "bias", torch.bfloat16), (workspace, "workspace", torch.uint8),
                        (out, "out", torch.bfloat16)):
        _cuda(t, dt, name)
    _check(load().qs_linear_bgr(_p(x), M, K, float(alpha), _p(w_packed), _p(w_scale),
                                _p(w_offset), _p(bias), N, bits, _p(workspace), workspace_bytes,
                                _p(out), _s(stream)), "qs_linear_bgr")


def qs_sd4_quant(x, rows, K, codes, meta, stream=None):
    _cuda(x, torch.bfloat16, "x")
    _cuda(codes, torch.uint8, "codes")
    _cuda(meta, torch.int16, "meta")
    _check(load().qs_sd4_quant(_p(x), rows, K, _p(codes), _p(meta), _s(stream)), "qs_sd4_quant")


def qs_sd4_linear(x_codes, x_meta, w_codes, w_meta, bias, M, N, K, out, stream=None):
    for t, name, dt in ((x_codes, "x_codes", torch.uint8), (w_codes, "w_codes", torch.uint8),
                        (x_meta, "x_meta", torch.int16), (w_meta, "w_meta", torch.int16),
                        (bias, "bias", torch.bfloat16), (out, "out", torch.bfloat16)):
        _cuda(t, dt, name)
    _check(load().qs_sd4_linear(_p(x_codes), _p(x_meta), _p(w_codes), _p(w_meta), _p(bias), M, N,
                                K, _p(out), _s(stream)), "qs_sd4_linear")


def sd4_linear(x_codes, x_meta, w_codes, w_meta, bias, K: int, stream=None, out=None):
    M, N = x_codes.shape[0], w_codes.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x_codes.device)
    qs_sd4_linear(x_codes, x_meta, w_codes, w_meta, bias, M, N, K, out, stream)
    return out


def qs_sd4_decode(codes, meta, rows, K, out, stream=None):
    _cuda(codes, torch.uint8, "codes")
    _cuda(meta, torch.int16, "meta")
    _cuda(out, torch.bfloat16, "out")
    _check(load().qs_sd4_decode(_p(codes), _p(meta), rows, K, _p(out), _s(stream)), "qs_sd4_decode")


def qs_sd4_linear_wdec(x_codes, x_meta, w, bias, M, N, K, out, stream=None):
    for t, name, dt in ((x_codes, "x_codes", torch.uint8), (x_meta, "x_meta", torch.int16),
                        (w, "w", torch.bfloat16), (bias, "bias", torch.bfloat16),
                        (out, "out", torch.bfloat16)):
        _cuda(t, dt, name)
    _check(load().qs_sd4_linear_wdec(_p(x_codes), _p(x_meta), _p(w), _p(bias), M, N, K, _p(out),
                                     _s(stream)), "qs_sd4_linear_wdec")


def sd4_decode(codes, meta, stream=None):
    R, K = codes.shape[0], codes.shape[1] * 2
    out = torch.empty((R, K), dtype=torch.bfloat16, device=codes.device)
    qs_sd4_decode(codes, meta, R, K, out, stream)
    return out


def sd4_quant(x: torch.Tensor, stream=None):
    """x bf16 [R, K] -> (codes uint8 [R, K/2], meta int16 [R, K/32]: e | d << 8)."""
    R, K = x.shape
    codes = torch.empty((R, K // 2), dtype=torch.uint8, device=x.device)
    meta = torch.empty((R, K // 32), dtype=torch.int16, device=x.device)
    qs_sd4_quant(x, R, K, codes, meta, stream)
    return codes, meta


def qs_sd4_quant_decomp(x, M, K, rows, S, codes2, meta2, stream=None):
    _cuda(x, torch.bfloat16, "x")
    _cuda(rows, torch.int32, "rows")
    _cuda(codes2, torch.uint8, "codes2")
    _cuda(meta2, torch.int16, "meta2")
    _check(load().qs_sd4_quant_decomp(_p(x), M, K, _p(rows), S, _p(codes2), _p(meta2),
                                      _s(stream)), "qs_sd4_quant_decomp")


def qs_sd4_linear_decomp(codes2, meta2, rows, S, w_codes, w_meta, w_e4m3, bias, M, N, K, out,
                         stream=None):
    for t, name, dt in ((codes2, "codes2", torch.uint8), (meta2, "meta2", torch.int16),
                        (rows, "rows", torch.int32), (w_codes, "w_codes", torch.uint8),
                        (w_meta, "w_meta", torch.int16), (w_e4m3, "w_e4m3", torch.uint8),
                        (bias, "bias", torch.bfloat16), (out, "out", torch.bfloat16)):
        _cuda(t, dt, name)
    _check(load().qs_sd4_linear_decomp(_p(codes2), _p(meta2), _p(rows), S, _p(w_codes),
                                       _p(w_meta), _p(w_e4m3), _p(bias), M, N, K, _p(out),
                                       _s(stream)), "qs_sd4_linear_decomp")


def qs_sd4_decode_e4m3(codes, meta, rows, K, out, stream=None):
    _cuda(codes, torch.uint8, "codes")
    _cuda(meta, torch.int16, "meta")
    _cuda(out, torch.uint8, "out")
    _check(load().qs_sd4_decode_e4m3(_p(codes), _p(meta), rows, K, _p(out), _s(stream)),
           "qs_sd4_decode_e4m3")


def sd4_decode_e4m3(codes, meta, stream=None):
    """SD4 codes [R, K/2] + block words -> e4m3 bytes uint8 [R, K] (the block
    scales stay in the words)."""
    R, K = codes.shape[0], codes.shape[1] * 2
    out = torch.empty((R, K), dtype=torch.uint8, device=codes.device)
    qs_sd4_decode_e4m3(codes, meta, R, K, out, stream)
    return out


def qs_sd4_linear_e4m3w(x_codes, x_meta, w_e4m3, w_meta, bias, M, N, K, out, stream=None):
    for t, name, dt in ((x_codes, "x_codes", torch.uint8), (x_meta, "x_meta", torch.int16),
                        (w_e4m3, "w_e4m3", torch.uint8), (w_meta, "w_meta", torch.int16),
                        (bias, "bias", torch.bfloat16), (out, "out", torch.bfloat16)):
        _cuda(t, dt, name)
    _check(load().qs_sd4_linear_e4m3w(_p(x_codes), _p(x_meta), _p(w_e4m3), _p(w_meta), _p(bias),
                                      M, N, K, _p(out), _s(stream)), "qs_sd4_linear_e4m3w")


def sd4_quant_decomp(x: torch.Tensor, rows: torch.Tensor, stream=None):
    """Salient rows `rows` (int32 [S]) of x bf16 [M, K] -> (codes2 uint8 [S, K],
    meta2 int16 [S, K/16]): [Q(x) | Q(x - x_hat)] per row."""
    M, K = x.shape
    S = rows.shape[0]
    codes2 = torch.empty((S, K), dtype=torch.uint8, device=x.device)
    meta2 = torch.empty((S, K // 16), dtype=torch.int16, device=x.device)
    qs_sd4_quant_decomp(x, M, K, rows, S, codes2, meta2, stream)
    return codes2, meta2


def sd4_linear_decomp(x_codes, x_meta, codes2, meta2, rows, w_codes, w_meta, bias, K: int,
                      w_e4m3=None, stream=None, out=None):
    """The SD4 layer with the salient rows decomposed: qs_sd4_linear (or the
    e4m3-weight form when w_e4m3 is given) over all rows, then
    qs_sd4_linear_decomp over the salient ones."""
    M, N = x_codes.shape[0], w_meta.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x_codes.device)
    if w_e4m3 is not None:
        qs_sd4_linear_e4m3w(x_codes, x_meta, w_e4m3, w_meta, bias, M, N, K, out, stream)
    else:
        qs_sd4_linear(x_codes, x_meta, w_codes, w_meta, bias, M, N, K, out, stream)
    qs_sd4_linear_decomp(codes2, meta2, rows, rows.shape[0],
                         None if w_e4m3 is not None else w_codes, w_meta, w_e4m3, bias, M, N, K,
                         out, stream)
    return out


def qs_sd4_quant_e4m3(x, rows, K, out, meta, stream=None):
    _cuda(x, torch.bfloat16, "x")
    _cuda(out, torch.uint8, "out")
    _cuda(meta, torch.int16, "meta")
    _check(load().qs_sd4_quant_e4m3(_p(x), rows, K, _p(out), _p(meta), _s(stream)),
           "qs_sd4_quant_e4m3")


def sd4_quant_e4m3(x: torch.Tensor, stream=None):
    """x bf16 [R, K] -> (e4m3 bytes uint8 [R, K], meta int16 [R, K/32])."""
    R, K = x.shape
    out = torch.empty((R, K), dtype=torch.uint8, device=x.device)
    meta = torch.empty((R, K // 32), dtype=torch.int16, device=x.device)
    qs_sd4_quant_e4m3(x, R, K, out, meta, stream)
    return out, meta


def qs_sd4_linear_e4m3(x_e4m3, x_meta, w_e4m3, w_meta, bias, M, N, K, out, stream=None):
    for t, name, dt in ((x_e4m3, "x_e4m3", torch.uint8), (x_meta, "x_meta", torch.int16),
                        (w_e4m3, "w_e4m3", torch.uint8), (w_meta, "w_meta", torch.int16),
                        (bias, "bias", torch.bfloat16), (out, "out", torch.bfloat16)):
        _cuda(t, dt, name)
    _check(load().qs_sd4_linear_e4m3(_p(x_e4m3), _p(x_meta), _p(w_e4m3), _p(w_meta), _p(bias),
                                     M, N, K, _p(out), _s(stream)), "qs_sd4_linear_e4m3")


def qs_sd4_scale_tiles_bytes(rows: int, K: int, weights: int) -> int:
    return int(load().qs_sd4_scale_tiles_bytes(rows, K, weights))


def qs_sd4_scale_tiles(meta, rows, K, weights, tiles, stream=None):
    _cuda(meta, torch.int16, "meta")
    _cuda(tiles, torch.uint8, "tiles")
    _check(load().qs_sd4_scale_tiles(_p(meta), rows, K, weights, _p(tiles), tiles.numel(),
                                     _s(stream)), "qs_sd4_scale_tiles")


def sd4_scale_tiles(meta: torch.Tensor, weights: bool, stream=None) -> torch.Tensor:
    """Block words [rows, K/32] -> the GEMM's pre-arranged scale tiles (uint8)."""
    rows, K = meta.shape[0], meta.shape[1] * 32
    need = qs_sd4_scale_tiles_bytes(rows, K, int(weights))
    if need < 0:
        raise QSError(2, f"qs_sd4_scale_tiles_bytes({rows}, {K})")
    tiles = torch.empty((need,), dtype=torch.uint8, device=meta.device)
    qs_sd4_scale_tiles(meta, rows, K, int(weights), tiles, stream)
    return tiles


def qs_sd4_linear_e4m3_tiles(x_e4m3, x_tiles, w_e4m3, w_tiles, bias, M, N, K, out, stream=None):
    for t, name, dt in ((x_e4m3, "x_e4m3", torch.uint8), (x_tiles, "x_tiles", torch.uint8),
                        (w_e4m3, "w_e4m3", torch.uint8), (w_tiles, "w_tiles", torch.uint8),
                        (bias, "bias", torch.bfloat16), (out, "out", torch.bfloat16)):
        _cuda(t, dt, name)
    _check(load().qs_sd4_linear_e4m3_tiles(_p(x_e4m3), _p(x_tiles), _p(w_e4m3), _p(w_tiles),
                                           _p(bias), M, N, K, _p(out), _s(stream)),
           "qs_sd4_linear_e4m3_tiles")


def qs_gbs_reset(state, stream=None):
    _cuda(state, torch.uint8, "state")
    _check(load().qs_gbs_reset(_p(state), _s(stream)), "qs_gbs_reset")


def qs_gbs_update(y_cur, y_prev, n, delta, state, stream=None):
    _cuda(y_cur, torch.bfloat16, "y_cur")
    _cuda(y_prev, torch.bfloat16, "y_prev")
    _cuda(state, torch.uint8, "state")
    _check(load().qs_gbs_update(_p(y_cur), _p(y_prev), n, float(delta), _p(state), _s(stream)),
           "qs_gbs_update")


def qs_linear_gbs(x, M, K, alpha, w4_packed, w4_scale, w8_packed, w8_scale, bias, N, state,
                  workspace, workspace_bytes, out, stream=None):
    _cuda(x, torch.bfloat16, "x")
    for t, name in ((w4_packed, "w4_packed"), (w8_packed, "w8_packed"), (state, "state"),
                    (workspace, "workspace")):
        _cuda(t, torch.uint8, name)
    _cuda(w4_scale, torch.float32, "w4_scale")
    _cuda(w8_scale, torch.float32, "w8_scale")
    _cuda(bias, torch.bfloat16, "bias")
    _cuda(out, torch.bfloat16, "out")
    _check(load().qs_linear_gbs(_p(x), M, K, float(alpha), _p(w4_packed), _p(w4_scale),
                                _p(w8_packed), _p(w8_scale), _p(bias), N, _p(state),
                                _p(workspace), workspace_bytes, _p(out), _s(stream)),
           "qs_linear_gbs")


def qs_selftest_timeout(timeout_us: int, stream=None) -> None:
    _check(load().qs_selftest_timeout(timeout_us, _s(stream)), "qs_selftest_timeout")


def qs_device_error(stream=None) -> int:
    return int(load().qs_device_error(_s(stream)))


def qs_version() -> str:
    return load().qs_version().decode()


# --------------------------------------------------------------------------- helpers

def packed_cols(K: int, bits: int, flags: int = 0) -> int:
    """Bytes of one packed row of K codes: nibbles for 4 bits (bytes with
    QS_FLAG_BYTE_CODES), bytes for 6 and 8."""
    return K // 2 if bits == 4 and not (flags & QS_FLAG_BYTE_CODES) else K


def storage_bits(bits: int, flags: int = 0) -> int:
    """The width the GEMM calls take for codes of `bits` written with `flags`."""
    return 8 if (flags & QS_FLAG_BYTE_CODES) else bits


def pack_weights(w: torch.Tensor, bits: int, flags: int = 0, stream=None):
    """w bf16 [N, K] -> (w_packed uint8 [N, packed_cols(K, bits)], w_scale float32 [N])."""
    N, K = w.shape
    wp = torch.empty((N, packed_cols(K, bits, flags)), dtype=torch.uint8, device=w.device)
    ws = torch.empty((N,), dtype=torch.float32, device=w.device)
    qs_pack_weights(w, N, K, bits, flags, wp, ws, stream)
    return wp, ws


def pack_weights_bgr(w: torch.Tensor, bits: int, candidates: int = 64, iterations: int = 8,
                     flags: int = 0, stream=None):
    """w bf16 [N, K] -> (signed codes on BGR grids, scales float32 [N], offsets int32 [N])."""
    N, K = w.shape
    wp = torch.empty((N, packed_cols(K, bits)), dtype=torch.uint8, device=w.device)
    ws = torch.empty((N,), dtype=torch.float32, device=w.device)
    wo = torch.empty((N,), dtype=torch.int32, device=w.device)
    qs_pack_weights_bgr(w, N, K, bits, flags, candidates, iterations, wp, ws, wo, stream)
    return wp, ws, wo


def quant_act_rowsum(x: torch.Tensor, bits: int, alpha: float = 1.0, flags: int = 0,
                     stream=None):
    """x bf16 [M, K] -> (packed codes, scales, per-token code sums int32 [M])."""
    M, K = x.shape
    xp = torch.empty((M, packed_cols(K, bits)), dtype=torch.uint8, device=x.device)
    xs = torch.empty((M,), dtype=torch.float32, device=x.device)
    xr = torch.empty((M,), dtype=torch.int32, device=x.device)
    qs_quant_act_rowsum(x, M, K, bits, alpha, flags, xp, xs, xr, stream)
    return xp, xs, xr


def quant_act(x: torch.Tensor, bits: int, alpha: float = 1.0, flags: int = 0, stream=None,
              out=None):
    """x bf16 [M, K] -> (x_packed uint8 [M, packed_cols(K, bits)], x_scale float32 [M])."""
    M, K = x.shape
    if out is None:
        xp = torch.empty((M, packed_cols(K, bits, flags)), dtype=torch.uint8, device=x.device)
        xs = torch.empty((M,), dtype=torch.float32, device=x.device)
    else:
        xp, xs = out
    qs_quant_act(x, M, K, bits, alpha, flags, xp, xs, stream)
    return xp, xs


def qlinear(x_packed, x_scale, w_packed, w_scale, bias, bits: int, K: int, stream=None, out=None,
            bits_w: int | None = None):
    """Packed activations (``bits``) and weights (``bits_w``, default ``bits``) -> bf16 [M, N]."""
    M, N = x_packed.shape[0], w_packed.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x_packed.device)
    if bits_w is None or bits_w == bits:
        qs_qlinear(x_packed, x_scale, w_packed, w_scale, bias, M, N, K, bits, out, stream)
    else:
        qs_qlinear_mixed(x_packed, x_scale, bits, w_packed, w_scale, bits_w, bias, M, N, K, out,
                         stream)
    return out


def qgemm_s32(x_packed, w_packed, bits: int, K: int, stream=None, bits_w: int | None = None):
    M, N = x_packed.shape[0], w_packed.shape[0]
    acc = torch.empty((M, N), dtype=torch.int32, device=x_packed.device)
    if bits_w is None or bits_w == bits:
        qs_qgemm_s32(x_packed, w_packed, M, N, K, bits, acc, stream)
    else:
        qs_qgemm_s32_mixed(x_packed, bits, w_packed, bits_w, M, N, K, acc, stream)
    return acc


def gelu(x: torch.Tensor, stream=None, out=None):
    y = torch.empty_like(x) if out is None else out
    qs_gelu_bf16(x, x.numel(), y, stream)
    return y


def linear(x, w_packed, w_scale, bias, bits: int, alpha: float = 1.0, workspace=None,
           stream=None, out=None, bits_w: int | None = None, x_flags: int = 0):
    """bf16 activations [M, K] -> bf16 [M, N] through one C call; ``bits`` is
    the activation width, ``bits_w`` the weights' storage width (default
    ``bits``), ``x_flags`` the activation quantisation flags."""
    M, K = x.shape
    N = w_packed.shape[0]
    need = qs_linear_workspace_bytes(M, K, storage_bits(bits, x_flags))
    if need < 0:
        raise QSError(2, "qs_linear_workspace_bytes")
    if workspace is None:
        workspace = torch.empty((need,), dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if x_flags:
        qs_linear_ex(x, M, K, alpha, bits, x_flags, w_packed, w_scale,
                     bits if bits_w is None else bits_w, bias, N, workspace, workspace.numel(),
                     out, stream)
    elif bits_w is None or bits_w == bits:
        qs_linear(x, M, K, alpha, w_packed, w_scale, bias, N, bits, workspace, workspace.numel(),
                  out, stream)
    else:
        qs_linear_mixed(x, M, K, alpha, bits, w_packed, w_scale, bits_w, bias, N, workspace,
                        workspace.numel(), out, stream)
    return out


class QuantLinear:
    """A Hadamard-rotated quantized linear layer (W4A4, W8A8, or mixed such as
    W4A8 / W4A6 with ``bits_x``): weights packed once; each call runs the
    one-call layer (the activation kernel, then the GEMM) on a workspace the
    layer keeps and grows as needed.  ``act_codes`` stores 4-bit activation
    codes two per byte ("packed", packed int4 widened in the GEMM's shared
    memory; the faster form with the GEMM's 256 x 512 tiles) or one per byte
    ("bytes", loaded by TMA straight into the operand tiles); the codes, and
    so the outputs, are the same."""

    def __init__(self, weight: torch.Tensor, bias: torch.Tensor | None, bits: int,
                 alpha: float = 1.0, bits_x: int | None = None, act_codes: str = "packed"):
        if act_codes not in ("bytes", "packed"):
            raise ValueError("act_codes is 'bytes' or 'packed'")
        self.N, self.K = weight.shape
        self.bits = bits
        self.bits_x = bits if bits_x is None else bits_x
        self.alpha = alpha
        self.x_flags = QS_FLAG_BYTE_CODES if (self.bits_x == 4 and act_codes == "bytes") else 0
        self.w_packed, self.w_scale = pack_weights(weight, bits)
        self.bias = bias
        self.workspace = None

    def __call__(self, x: torch.Tensor, stream=None, out=None) -> torch.Tensor:
        need = qs_linear_workspace_bytes(x.shape[0], self.K, storage_bits(self.bits_x, self.x_flags))
        if self.workspace is None or self.workspace.numel() < need:
            self.workspace = torch.empty((max(need, 0),), dtype=torch.uint8, device=x.device)
        return linear(x, self.w_packed, self.w_scale, self.bias, self.bits_x, self.alpha,
                      self.workspace, stream=stream, out=out, bits_w=self.bits,
                      x_flags=self.x_flags)


def gbs_state_host(state) -> dict:
    """Copies the header of a qs_gbs_state to the host (synchronises)."""
    import struct
    raw = bytes(state[:32].cpu().numpy().tobytes())
    acc, last_d, bits, step, blocks_done, _ = struct.unpack("<ddiiII", raw)
    return {"acc": acc, "last_d": last_d, "bits": bits, "step": step, "blocks_done": blocks_done}


class GbsLinear:
    """A layer under δ-guided bit switching: weights quantised at 4 bits (codes
    stored one per byte, the form qs_linear_gbs takes) and at 8 bits, one
    device-side state; each call runs the layer at the width the state holds
    and then measures the change of its output against the previous call's,
    choosing the next width on the device (no host synchronisation)."""

    def __init__(self, weight: torch.Tensor, bias: torch.Tensor | None, delta: float,
                 alpha: float = 1.0, stream=None):
        self.N, self.K = weight.shape
        self.delta, self.alpha = float(delta), alpha
        self.w4, self.s4 = pack_weights(weight, 4, QS_FLAG_BYTE_CODES, stream=stream)
        self.w8, self.s8 = pack_weights(weight, 8, stream=stream)
        self.bias = bias
        self.state = torch.zeros((QS_GBS_STATE_BYTES,), dtype=torch.uint8, device=weight.device)
        qs_gbs_reset(self.state, stream)
        self.workspace = None
        self.prev = None
        self.buffers = []  # two outputs used in turn when the caller passes none

    def __call__(self, x: torch.Tensor, stream=None, out=None) -> torch.Tensor:
        M = x.shape[0]
        need = qs_linear_workspace_bytes(M, self.K, 8)
        if self.workspace is None or self.workspace.numel() < need:
            self.workspace = torch.empty((max(need, 0),), dtype=torch.uint8, device=x.device)
        if out is None:
            if not self.buffers or self.buffers[0].shape != (M, self.N):
                self.buffers = [torch.empty((M, self.N), dtype=torch.bfloat16, device=x.device)
                                for _ in range(2)]
            self.buffers.reverse()
            out = self.buffers[0]
        if self.prev is not None and out.data_ptr() == self.prev.data_ptr():
            raise ValueError("out must not be the previous step's output")
        qs_linear_gbs(x, M, self.K, self.alpha, self.w4, self.s4, self.w8, self.s8, self.bias,
                      self.N, self.state, self.workspace, self.workspace.numel(), out, stream)
        prev = self.prev if self.prev is not None and self.prev.shape == out.shape else None
        qs_gbs_update(out, prev, out.numel(), self.delta, self.state, stream)
        self.prev = out
        return out
