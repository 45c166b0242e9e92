"""Hadamard-rotated quantized linear layer (W4A4, W8A8, and the mixed W4A8 /
W4A6) for NVIDIA B200 (sm_100a).

The computation runs in libqs.so (CUDA kernels behind a C ABI, see include/qs.h);
this package holds its build script, a ctypes binding and the seeded synthetic
inputs used by the tests and the benchmark.
"""
from .binding import (  # noqa: F401
    BITS, EXPORTS, QS_FLAG_BYTE_CODES, QS_FLAG_NO_ROTATE, QS_GBS_STATE_BYTES, QS_MAX_K, GbsLinear, QSError,
    QuantLinear, gbs_state_host, gelu, linear, load, pack_weights_bgr, quant_act_rowsum,
    qs_gbs_reset, qs_gbs_update, qs_linear_bgr, qs_linear_bgr_workspace_bytes, qs_linear_gbs,
    qs_pack_weights_bgr, qs_qgemm_s32_asym, qs_qlinear_asym, qs_quant_act_rowsum, qs_linear_ex,
    storage_bits, qs_sd4_quant, sd4_quant, qs_sd4_linear, sd4_linear, qs_sd4_decode, sd4_decode,
    qs_sd4_linear_wdec, qs_sd4_quant_decomp, qs_sd4_linear_decomp, sd4_quant_decomp,
    sd4_linear_decomp, qs_sd4_decode_e4m3, sd4_decode_e4m3, qs_sd4_linear_e4m3w,
    qs_sd4_quant_e4m3, sd4_quant_e4m3, qs_sd4_linear_e4m3, qs_sd4_scale_tiles_bytes,
    qs_sd4_scale_tiles, sd4_scale_tiles, qs_sd4_linear_e4m3_tiles,
    pack_weights, packed_cols, qgemm_s32, qlinear, qs_device_error, qs_gelu_bf16, qs_linear,
    qs_linear_mixed, qs_linear_workspace_bytes, qs_pack_weights, qs_qgemm_s32, qs_qgemm_s32_mixed,
    qs_qlinear, qs_qlinear_mixed, qs_quant_act, qs_selftest_timeout, qs_version, quant_act,
)
