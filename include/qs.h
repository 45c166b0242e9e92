/*
 * qs.h — C ABI of libqs.so: the Hadamard-rotated W4A4 / W8A8 quantized linear
 * layer, and its mixed-width forms W4A8 / W4A6, on NVIDIA B200 (sm_100a).
 *
 * The layer follows DVD-Quant ("Data-free Video Diffusion Transformers
 * Quantization"), "Resumen técnico" §2.B, Auto-scaling Rotated Quantization:
 * a Hadamard rotation is applied to both activations and weights, and the
 * quantization scales are computed at run time from the rotated activations
 * (no calibration data).  The bit widths are W4A4 (§1, §4), the 8-bit branch
 * of δ-GBS (§2.C), W4A6 (DVD-Quant §4, the 6-bit activation setting) and
 * W4A8 (QuantSparse, "Resumen técnico" §4: 4-bit weights, 8-bit
 * activations).  Quantities the pages leave open are fixed here as follows:
 *   - rotation: Sylvester Hadamard of order 128 in natural order,
 *     H[i][j] = (-1)^popcount(i&j), on consecutive blocks of 128 along K,
 *     computed as the binary32 butterfly with stages h = 1,2,4,...,64;
 *   - the 1/sqrt(128) of each rotation is folded into the weight scale
 *     (both together are the exact factor 2^-7);
 *   - activations: one scale per token (row) over all of K, clip ratio alpha;
 *     weights: one scale per output channel (row of W), alpha = 1;
 *   - t = fl(alpha * amax); stored scale s = fl(t / qmax); multiplier
 *     inv = fl(qmax / t); qmax = 2^(bits-1) - 1: 7, 31 or 127 for 4, 6, 8 bits;
 *     q = clamp(round_half_even(u * inv), -qmax, qmax), the product exact and
 *     rounded once; rows with t < 2^-120 (amax == 0 included): s = 0, q = 0;
 *   - out = bf16_rne(fl(fl(fl(s_a[m] * s_w[n]) * float(acc[m][n])) + bias[n])),
 *     acc = sum_k q_a[m][k] * q_w[n][k] exact in int32.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers on the current CUDA device,
 *     16-byte aligned, owned and allocated by the caller.  The library
 *     allocates no memory and keeps no per-call state.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream); every
 *     call only enqueues work on it and returns without synchronising.
 *   - Arguments are validated before anything is launched; a call that
 *     returns anything but QS_OK has launched nothing.
 *   - No C++ exception crosses this interface.
 *
 * Packed formats (row-major; rows of K/2 bytes for 4 bits, K bytes otherwise)
 *   - 8 and 6 bits: one two's complement byte per element.
 *   - 4 bits: two's complement nibbles; byte j of a row holds element 2j in
 *     its low nibble and element 2j+1 in its high nibble.
 *   Codes are always in [-qmax, qmax].  `bits` arguments take 4, 6 or 8.
 */
#ifndef QS_H_
#define QS_H_

#include <stdint.h>

#if defined(__GNUC__)
#define QS_API __attribute__((visibility("default")))
#else
#define QS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QS_OK = 0,
  QS_ERR_NULL = 1,     /* a required pointer is NULL */
  QS_ERR_SHAPE = 2,    /* M, N or K <= 0, K % 128 != 0, or N % 16 != 0 */
  QS_ERR_BITS = 3,     /* bits not 4, 6 or 8 */
  QS_ERR_ALIGN = 4,    /* a pointer is not 16-byte aligned */
  QS_ERR_RANGE = 5,    /* alpha outside [2^-14, 1], unknown flag bits, a size above its limit,
                          or (from qs_device_error) a row index out of range */
  QS_ERR_CUDA = 6,     /* a CUDA runtime/driver call or a launch failed */
  QS_ERR_TIMEOUT = 7,  /* a kernel wait exceeded its bound (reported by qs_device_error) */
  QS_ERR_PTR = 8       /* a pointer is not device memory of the current device */
} qs_status;

/* Test-only flag: skip the Hadamard rotation (the codes are then taken from the
 * input values themselves, which makes rounding ties easy to construct). */
#define QS_FLAG_NO_ROTATE 1u
/* Storage flag for qs_quant_act / qs_pack_weights (and the _rowsum form):
 * 4-bit codes are written one per byte (int8, values in [-7, 7]) instead of
 * two per byte.  Such codes are passed to the GEMM calls with bits = 8 (the
 * GEMM only needs the storage; the accumulator bounds hold a fortiori).  For
 * activations this trades M*K/2 bytes of extra writes for a GEMM that loads
 * them by TMA straight into its operand tiles; the arithmetic is unchanged. */
#define QS_FLAG_BYTE_CODES 2u

/* Largest K accepted.  With |q| <= 127 the int32 accumulator cannot overflow
 * (127^2 * 65536 < 2^31), and the rotate-quantize kernel keeps a whole row in
 * registers in one pass up to this length. */
#define QS_MAX_K 65536
/* Largest M or N accepted (tensor-map coordinates are 32-bit). */
#define QS_MAX_ROWS 2147483647LL

/*
 * qs_pack_weights — offline weight preparation.
 * DVD-Quant §2.B: the Hadamard rotation is applied to the weights as well as
 * to the activations.  Rotates every row of W along K, quantizes it with its
 * own scale (one per output channel, alpha = 1) and packs it.
 *   w_bf16   [N, K] bf16, row-major (torch.nn.Linear layout; y = x W^T + b)
 *   bits     4, 6 or 8
 *   flags    QS_FLAG_NO_ROTATE, QS_FLAG_BYTE_CODES or both
 *   w_packed [N, K/2] bytes (4 bits, packed) or [N, K] bytes, written
 *   w_scale  [N] float, written: s * 2^-7 (or s with QS_FLAG_NO_ROTATE)
 */
QS_API qs_status qs_pack_weights(const void* w_bf16, int64_t N, int64_t K, int bits, unsigned flags,
                          void* w_packed, float* w_scale, void* stream);

/*
 * qs_quant_act — the fused activation kernel of the hot path.
 * DVD-Quant §2.B: rotate the activations with the Hadamard matrix, then scale
 * them with factors computed at run time from the rotated values.  Per token:
 * 128-point block Walsh-Hadamard transform along K, absmax, scale with clip
 * ratio alpha, round-half-even, pack.
 *   x_bf16   [M, K] bf16, row-major
 *   bits     4, 6 or 8
 *   alpha    clip ratio in [2^-14, 1]
 *   flags    QS_FLAG_NO_ROTATE, QS_FLAG_BYTE_CODES or both
 *   x_packed [M, K/2] bytes (4 bits, packed) or [M, K] bytes, written
 *   x_scale  [M] float, written (the per-token scale s_a)
 */
QS_API qs_status qs_quant_act(const void* x_bf16, int64_t M, int64_t K, int bits, float alpha,
                       unsigned flags, void* x_packed, float* x_scale, void* stream);

/*
 * qs_qlinear — integer tensor-core GEMM with the dequantizing epilogue.
 * The low-bit product of DVD-Quant's W4A4 (§1, §4) / 8-bit (§2.C) layers:
 * out[m][n] = bf16(s_a[m] * s_w[n] * sum_k q_a[m][k] q_w[n][k] + bias[n]).
 *   x_packed, x_scale  from qs_quant_act (same K and bits)
 *   w_packed, w_scale  from qs_pack_weights (same K and bits)
 *   bias_bf16          [N] bf16 or NULL (NULL adds +0.0)
 *   N % 16 == 0 is required; M is arbitrary.
 *   out_bf16           [M, N] bf16, row-major, written
 */
QS_API qs_status qs_qlinear(const void* x_packed, const float* x_scale, const void* w_packed,
                     const float* w_scale, const void* bias_bf16, int64_t M, int64_t N,
                     int64_t K, int bits, void* out_bf16, void* stream);

/*
 * qs_qlinear_mixed — qs_qlinear with the activation codes at `bits_x` and the
 * weight codes at `bits_w` (each 4, 6 or 8): W4A8 is bits_x = 8, bits_w = 4
 * (QuantSparse §4), W4A6 is bits_x = 6, bits_w = 4 (DVD-Quant §4).  Same
 * arithmetic and output as qs_qlinear; qs_qlinear(..., bits, ...) is this
 * call with bits_x = bits_w = bits.
 *   x_packed, x_scale  from qs_quant_act at bits_x
 *   w_packed, w_scale  from qs_pack_weights at bits_w
 *   other arguments as qs_qlinear
 */
QS_API qs_status qs_qlinear_mixed(const void* x_packed, const float* x_scale, int bits_x,
                                  const void* w_packed, const float* w_scale, int bits_w,
                                  const void* bias_bf16, int64_t M, int64_t N, int64_t K,
                                  void* out_bf16, void* stream);

/*
 * qs_qgemm_s32 — the same GEMM main loop with an int32 epilogue: writes the
 * exact accumulators acc[m][n] = sum_k q_a[m][k] q_w[n][k] (parity checks).
 *   acc [M, N] int32, row-major, written.  N % 16 == 0.
 */
QS_API qs_status qs_qgemm_s32(const void* x_packed, const void* w_packed, int64_t M, int64_t N,
                       int64_t K, int bits, int32_t* acc, void* stream);

/* qs_qgemm_s32_mixed — qs_qgemm_s32 with separate code widths (as qs_qlinear_mixed). */
QS_API qs_status qs_qgemm_s32_mixed(const void* x_packed, int bits_x, const void* w_packed,
                                    int bits_w, int64_t M, int64_t N, int64_t K, int32_t* acc,
                                    void* stream);

/*
 * qs_linear_workspace_bytes — bytes of device scratch that qs_linear needs for
 * M tokens of K inputs with activation codes of `bits`: the packed activations
 * (M*K/2 bytes for 4 bits, M*K otherwise, rounded up to 256) followed by the
 * per-token scales (4*M bytes).  Returns -1 for arguments qs_linear would
 * reject.
 */
QS_API int64_t qs_linear_workspace_bytes(int64_t M, int64_t K, int bits);

/*
 * qs_linear — the whole layer in one call: qs_quant_act into the caller's
 * workspace, then qs_qlinear (DVD-Quant §2.B: rotate and scale the
 * activations at run time, then the low-bit product).  Results are identical
 * to calling the two entry points in sequence.
 *   x_bf16             [M, K] bf16
 *   alpha              clip ratio in [2^-14, 1]
 *   w_packed, w_scale  from qs_pack_weights (same K and bits)
 *   bias_bf16          [N] bf16 or NULL
 *   workspace          device scratch of at least qs_linear_workspace_bytes(M, K, bits)
 *                      bytes, 16-byte aligned; overwritten; must not overlap other arguments
 *   out_bf16           [M, N] bf16, written
 */
QS_API qs_status qs_linear(const void* x_bf16, int64_t M, int64_t K, float alpha,
                           const void* w_packed, const float* w_scale, const void* bias_bf16,
                           int64_t N, int bits, void* workspace, int64_t workspace_bytes,
                           void* out_bf16, void* stream);

/*
 * qs_linear_ex — qs_linear_mixed with quantisation flags for the activations
 * (0 or QS_FLAG_BYTE_CODES; the GEMM then reads 4-bit activation codes as
 * bytes).  The workspace is qs_linear_workspace_bytes(M, K, s) with s = 8 when
 * the activation codes are stored in bytes, else bits_x.
 */
QS_API qs_status qs_linear_ex(const void* x_bf16, int64_t M, int64_t K, float alpha, int bits_x,
                              unsigned x_flags, const void* w_packed, const float* w_scale,
                              int bits_w, const void* bias_bf16, int64_t N, void* workspace,
                              int64_t workspace_bytes, void* out_bf16, void* stream);

/*
 * qs_linear_mixed — qs_linear with the activations quantized at `bits_x` and
 * weights packed at `bits_w` (W4A8: 8 and 4; W4A6: 6 and 4).  The workspace
 * is qs_linear_workspace_bytes(M, K, bits_x).
 */
QS_API qs_status qs_linear_mixed(const void* x_bf16, int64_t M, int64_t K, float alpha,
                                 int bits_x, const void* w_packed, const float* w_scale,
                                 int bits_w, const void* bias_bf16, int64_t N, void* workspace,
                                 int64_t workspace_bytes, void* out_bf16, void* stream);

/*
 * Bounded-init grid refinement of the weights (DVD-Quant "Resumen técnico"
 * §2.A): per output channel an asymmetric b-bit grid (step Δ, integer zero
 * point z, levels 0..2^b-1) for the rotated weight row u, found offline by a
 * bound search that progressively excludes outliers followed by closed-form
 * least-squares refits of Δ and z.  Readings (the pages give no formula or
 * count): candidate bounds r_j [min u, max u], r_j = 1 - j/(2J), j < J, each
 * giving Δ = (hi - lo)/(2^b - 1) and z = clamp(rint(-lo/Δ)); the smallest
 * squared error wins; then T refits: least squares u ≈ Δ q + c on the current
 * codes, z = clamp(rint(-c/Δ)), Δ refit for that z, keep the best grid.  Codes
 * q = clamp(rint(u * fl(1/Δ)) + z, 0, 2^b - 1); every sum in index order in
 * binary64.  Stored: signed codes s = q - 2^(b-1) (same packing as the
 * symmetric path: nibbles or bytes), scale fl32(Δ) * 2^-7 (the rotations'
 * normalisation, as in qs_pack_weights) and offset o = 2^(b-1) - z, so that
 * Δ (q - z) = Δ (s + o).  The layer's accumulator is then
 * sum_k q_a s + o[n] * sum_k q_a[m,k] (exact in int32).
 */

/*
 * qs_pack_weights_bgr — offline: rotate every row of W (unless
 * QS_FLAG_NO_ROTATE), choose its grid as above and pack it.
 *   w_bf16      [N, K] bf16; K <= 32768 (the row is held on chip)
 *   bits        4 or 8
 *   candidates  J in 1..256;  iterations  T in 0..64  (64 and 8 are typical)
 *   w_packed    [N, K/2] (4 bits) or [N, K] bytes, written
 *   w_scale     [N] float, written;  w_offset  [N] int32, written
 */
QS_API qs_status qs_pack_weights_bgr(const void* w_bf16, int64_t N, int64_t K, int bits,
                                     unsigned flags, int candidates, int iterations,
                                     void* w_packed, float* w_scale, int32_t* w_offset,
                                     void* stream);

/*
 * qs_quant_act_rowsum — qs_quant_act that also writes every token's code sum
 * x_rowsum[m] = sum_k q_a[m,k] (int32 [M]; zeroed and filled by the call),
 * which the asymmetric weight grid needs.
 */
QS_API qs_status qs_quant_act_rowsum(const void* x_bf16, int64_t M, int64_t K, int bits,
                                     float alpha, unsigned flags, void* x_packed,
                                     float* x_scale, int32_t* x_rowsum, void* stream);

/*
 * qs_qlinear_asym — qs_qlinear for weights from qs_pack_weights_bgr:
 * out = bf16(fl(fl(fl(s_a s_w) * float(acc)) + bias)) with
 * acc = sum_k q_a s + o[n] * x_rowsum[m].  bits 4 or 8 (both operands).
 */
QS_API qs_status qs_qlinear_asym(const void* x_packed, const float* x_scale,
                                 const int32_t* x_rowsum, const void* w_packed,
                                 const float* w_scale, const int32_t* w_offset,
                                 const void* bias_bf16, int64_t M, int64_t N, int64_t K,
                                 int bits, void* out_bf16, void* stream);

/* qs_qgemm_s32_asym — the exact accumulators of qs_qlinear_asym (parity checks). */
QS_API qs_status qs_qgemm_s32_asym(const void* x_packed, const int32_t* x_rowsum,
                                   const void* w_packed, const int32_t* w_offset, int64_t M,
                                   int64_t N, int64_t K, int bits, int32_t* acc, void* stream);

/*
 * qs_linear_bgr — the one-call layer for BGR weights: qs_quant_act_rowsum into
 * the workspace, then qs_qlinear_asym.  The workspace holds the packed
 * activations, the scales and the code sums:
 * qs_linear_bgr_workspace_bytes(M, K, bits) bytes (-1 for rejected arguments).
 */
QS_API int64_t qs_linear_bgr_workspace_bytes(int64_t M, int64_t K, int bits);
QS_API qs_status qs_linear_bgr(const void* x_bf16, int64_t M, int64_t K, float alpha,
                               const void* w_packed, const float* w_scale,
                               const int32_t* w_offset, const void* bias_bf16, int64_t N,
                               int bits, void* workspace, int64_t workspace_bytes,
                               void* out_bf16, void* stream);

/*
 * SD4 (SemanticDialect "Resumen técnico" §2.A, mixed-format 4-bit blocks):
 * each block of 32 consecutive elements of a row gets a power-of-two scale
 * 2^e that normalises its magnitudes to [0, 2) and the one of 32 4-bit
 * formats ("dialects") that fits it best, chosen through precomputed tables.
 * The pages print no dialect values; this library's formatbook: a code is a
 * sign bit (bit 3) and a level index i (bits 0-2); dialect d = 8a + s has the
 * magnitudes L/8 with L0 = 0, top level t = 15 - a and, for i = 1..7,
 * L = floor((2t(49p i + 7q i^2 + r i^3) + 2744) / 5488) made strictly
 * increasing, (p,q,r) = shape s of (8,0,0) (6,2,0) (4,4,0) (3,5,0) (2,5,1)
 * (0,8,0) (1,3,4) (0,3,5).  Block: e = max(floor(log2 amax), -126) (0 for a
 * zero block); bin b = min(floor(|x| 2^(7-e)), 255); Qerror[d][b] =
 * min_i (2b + 1 - 32 L_i)^2 and Qvalue[d][b] the minimising i; the block's
 * dialect minimises sum Qerror (smallest d on ties); code = sign | Qvalue.
 * Decoded value: (-1)^sign L/8 2^e (exact in bf16).
 */

/*
 * qs_sd4_quant — SD4 codes of a bf16 matrix (activations or weights).
 *   x_bf16  [rows, K] bf16, K % 256 == 0
 *   codes   [rows, K/2] bytes, written: element 2j in the low nibble of byte j
 *   meta    [rows, K/32] uint16, written: low byte e (int8), high byte d
 */
QS_API qs_status qs_sd4_quant(const void* x_bf16, int64_t rows, int64_t K, void* codes,
                              uint16_t* meta, void* stream);

/*
 * qs_sd4_quant_e4m3 — qs_sd4_quant with each element written as the e4m3
 * byte of its decoded magnitude and sign (the same values: (-1)^s L/8; the
 * block words, identical to qs_sd4_quant's, keep the block scales).  One byte
 * per element instead of half: the activation form that
 * qs_sd4_linear_e4m3 loads by TMA straight into its operand tiles.
 *   out_e4m3  [rows, K] bytes, written;  meta [rows, K/32] uint16, written
 */
QS_API qs_status qs_sd4_quant_e4m3(const void* x_bf16, int64_t rows, int64_t K, void* out_e4m3,
                                   uint16_t* meta, void* stream);

/*
 * qs_sd4_linear — the SD4 layer: out[m][n] = bf16(fl(sum_k x_hat w_hat) + bias[n])
 * with x_hat, w_hat the decoded SD4 values of qs_sd4_quant(x) and
 * qs_sd4_quant(W).  Each decoded value is an e4m3 number (L/8, signed) times
 * its block's power of two, so the product runs on the block-scaled fp8
 * tensor-core path (one UE8M0 scale per 32 elements along K): the products
 * are exact and summed with binary32 accumulation (parity is checked within
 * that bound).  K % 256 == 0, N % 16 == 0; bias NULL adds +0.0.
 *   out_bf16  [M, N] bf16, written
 */
QS_API qs_status qs_sd4_linear(const void* x_codes, const uint16_t* x_meta, const void* w_codes,
                               const uint16_t* w_meta, const void* bias_bf16, int64_t M,
                               int64_t N, int64_t K, void* out_bf16, void* stream);

/*
 * qs_sd4_decode — the decoded values of an SD4 matrix, bf16 [rows, K] (exact).
 * Offline use: decoding the weights once lets qs_sd4_linear_wdec load them by
 * TMA straight into the GEMM's operand tiles (only the activations are then
 * decoded per call), at 2 bytes per weight instead of half a byte.
 */
QS_API qs_status qs_sd4_decode(const void* codes, const uint16_t* meta, int64_t rows, int64_t K,
                               void* out_bf16, void* stream);

/*
 * qs_sd4_linear_wdec — the SD4 layer with the weights given decoded to bf16
 * (qs_sd4_decode of qs_sd4_quant(W)), on the bf16 tensor-core path (the
 * activations decoded to bf16 in the kernel).  The same exact products with
 * binary32 accumulation as qs_sd4_linear (outputs may differ from it only by
 * the accumulation order).  w_bf16 [N, K].
 */
QS_API qs_status qs_sd4_linear_wdec(const void* x_codes, const uint16_t* x_meta,
                                    const void* w_bf16, const void* bias_bf16, int64_t M,
                                    int64_t N, int64_t K, void* out_bf16, void* stream);

/*
 * qs_sd4_decode_e4m3 — the e4m3 bytes of an SD4 matrix: element k of a row
 * is the e4m3 encoding of its signed L/8 (exact); the block words keep the
 * block scales.  Offline use for the weights: qs_sd4_linear_e4m3w then loads
 * them by TMA straight into the GEMM's operand tiles, at one byte per weight.
 *   codes [rows, K/2], meta [rows, K/32] (qs_sd4_quant); out_e4m3 [rows, K] bytes
 */
QS_API qs_status qs_sd4_decode_e4m3(const void* codes, const uint16_t* meta, int64_t rows,
                                    int64_t K, void* out_e4m3, void* stream);

/*
 * qs_sd4_linear_e4m3w — qs_sd4_linear with the weights given as
 * qs_sd4_decode_e4m3 bytes (w_e4m3 [N, K]) and their block words
 * (w_meta [N, K/32]); only the activations are decoded per call.  The same
 * arithmetic as qs_sd4_linear.
 */
QS_API qs_status qs_sd4_linear_e4m3w(const void* x_codes, const uint16_t* x_meta,
                                     const void* w_e4m3, const uint16_t* w_meta,
                                     const void* bias_bf16, int64_t M, int64_t N, int64_t K,
                                     void* out_bf16, void* stream);

/*
 * qs_sd4_linear_e4m3 — qs_sd4_linear with both operands as e4m3 bytes and
 * block words (x from qs_sd4_quant_e4m3, W from qs_sd4_decode_e4m3 or
 * qs_sd4_quant_e4m3): nothing is decoded in the GEMM.  The same arithmetic
 * as qs_sd4_linear.
 *   x_e4m3 [M, K], x_meta [M, K/32], w_e4m3 [N, K], w_meta [N, K/32]
 */
QS_API qs_status qs_sd4_linear_e4m3(const void* x_e4m3, const uint16_t* x_meta,
                                    const void* w_e4m3, const uint16_t* w_meta,
                                    const void* bias_bf16, int64_t M, int64_t N, int64_t K,
                                    void* out_bf16, void* stream);

/*
 * qs_sd4_scale_tiles — the UE8M0 scale bytes (e + 127) of an SD4 matrix's
 * block words, arranged as the SD4 GEMM copies them into tensor memory, so
 * that qs_sd4_linear_e4m3_tiles loads them with the operands instead of
 * converting block words in the kernel.  Rows go in groups of 128
 * (weights = 0: activations) or 192 (weights = 1: one N-half of the GEMM's
 * 384-column tile; the group count is rounded up to even), each group padded
 * to 128 or 256 rows; per group and 128-element K step one tile of 512 or
 * 1024 bytes: row r of the group, 32-element block j of the step at byte
 * 512 (r / 128) + 16 (r % 32) + 4 ((r % 128) / 32) + j.  Padding rows are 0.
 *   meta   [rows, K/32] block words (qs_sd4_quant, qs_sd4_quant_e4m3)
 *   tiles  qs_sd4_scale_tiles_bytes(rows, K, weights) bytes, written;
 *          tiles_bytes: its size (QS_ERR_RANGE if smaller)
 * qs_sd4_scale_tiles_bytes returns -1 for an invalid shape.
 */
QS_API int64_t qs_sd4_scale_tiles_bytes(int64_t rows, int64_t K, int weights);
QS_API qs_status qs_sd4_scale_tiles(const uint16_t* meta, int64_t rows, int64_t K, int weights,
                                    void* tiles, int64_t tiles_bytes, void* stream);

/*
 * qs_sd4_linear_e4m3_tiles — qs_sd4_linear_e4m3 with the scales given as
 * qs_sd4_scale_tiles of the activations (weights = 0) and of the weights
 * (weights = 1): the GEMM copies operands and scales, nothing else.  The same
 * arithmetic, bit-identical output.
 *   x_e4m3 [M, K], x_tiles, w_e4m3 [N, K], w_tiles; other arguments as
 *   qs_sd4_linear_e4m3
 */
QS_API qs_status qs_sd4_linear_e4m3_tiles(const void* x_e4m3, const void* x_tiles,
                                          const void* w_e4m3, const void* w_tiles,
                                          const void* bias_bf16, int64_t M, int64_t N, int64_t K,
                                          void* out_bf16, void* stream);

/*
 * Activation decomposition (SemanticDialect "Resumen técnico" §2.B): a salient
 * activation row A is split into its SD4 value Q(A) and the residual
 * Delta = A - x_hat, which is quantised again with the same format, and the
 * layer uses A ~ Q(A) + Q(Delta) for that row.  The pages choose the salient
 * rows from attention scores; here the caller gives them as row indices.
 *
 * qs_sd4_quant_decomp — the decomposed rows: row i of the output holds 2K
 * codes, the SD4 codes of x[rows[i]] (those qs_sd4_quant writes) followed by
 * the SD4 codes of Delta (exact in binary32; blocks of the same 32 columns),
 * and the 2K/32 block words.
 *   x_bf16  [M, K] bf16, K % 256 == 0, K <= QS_MAX_K / 2
 *   rows    [S] int32 (device, 4-byte aligned); indices may repeat; an index
 *           outside [0, M) gives zero codes and words for that row and makes
 *           qs_device_error report QS_ERR_RANGE
 *   codes2  [S, K] bytes (2K codes, two per byte), written
 *   meta2   [S, K/16] uint16 (2K/32 block words), written
 */
QS_API qs_status qs_sd4_quant_decomp(const void* x_bf16, int64_t M, int64_t K,
                                     const int32_t* rows, int64_t S, void* codes2,
                                     uint16_t* meta2, void* stream);

/*
 * qs_sd4_linear_decomp — the decomposed rows of the SD4 layer: for i < S,
 *   out[rows[i]][n] = bf16(fl(sum_k (x_hat + delta_hat)[k] w_hat[n][k]) + bias[n])
 * as one binary32 accumulation (block-scaled fp8 tensor cores, as
 * qs_sd4_linear) over the 2K products of a qs_sd4_quant_decomp row with
 * [w_hat | w_hat].  Only those rows of out are written: the layer with
 * decomposition is qs_sd4_linear (or _e4m3w) over all M rows followed, on the
 * same stream, by this call.  The weights: their block words w_meta
 * [N, K/32] and either their codes (w_codes [N, K/2]) or, when w_e4m3 is not
 * NULL, their qs_sd4_decode_e4m3 bytes ([N, K]; w_codes is then ignored).
 * An index outside [0, M) is skipped and reported as in qs_sd4_quant_decomp.
 *   out_bf16  [M, N] bf16, rows rows[i] written
 */
QS_API qs_status qs_sd4_linear_decomp(const void* codes2, const uint16_t* meta2,
                                      const int32_t* rows, int64_t S, const void* w_codes,
                                      const uint16_t* w_meta, const void* w_e4m3,
                                      const void* bias_bf16, int64_t M, int64_t N, int64_t K,
                                      void* out_bf16, void* stream);

/*
 * δ-guided bit switching (DVD-Quant "Resumen técnico" §2.C): per layer, the
 * normalised L1 change between consecutive outputs is accumulated, and the
 * layer's next step runs at 4 bits while the accumulated change is below
 * delta, otherwise at 8 bits with the accumulator reset.  The state lives in
 * caller-owned device memory and is read and written only by the library's
 * kernels, so choosing the width needs no host synchronisation.  Readings:
 * d = sum|y_cur - y_prev| / sum|y_prev| over all elements (binary64 terms and
 * sums; a zero denominator gives 0 if the outputs are equal, else +inf);
 * "below delta" is strict; the first step runs at 8 bits.
 *
 * qs_gbs_state — layout of the state (copy it to the host to inspect it).
 *   acc     accumulated change since the last switch to 8 bits
 *   last_d  distance measured by the last update (-1 after a reset or a first step)
 *   bits    width of the layer's next step: 4 or 8
 *   step    updates since the reset
 *   blocks_done, partial: scratch of the update kernel (must stay as the
 *           library leaves it: zero between calls)
 */
#define QS_GBS_MAX_BLOCKS 1024
typedef struct {
  double acc;
  double last_d;
  int32_t bits;
  int32_t step;
  uint32_t blocks_done;
  uint32_t reserved_;
  double partial[2][QS_GBS_MAX_BLOCKS];
} qs_gbs_state;

/* qs_gbs_reset — enqueues: acc = 0, last_d = -1, bits = 8, step = 0.
 *   state  device pointer to a qs_gbs_state, 16-byte aligned */
QS_API qs_status qs_gbs_reset(void* state, void* stream);

/*
 * qs_gbs_update — after a step of the layer: measures the change between its
 * output and the previous step's and decides the next step's width.
 *   y_cur_bf16   this step's output, n bf16 values
 *   y_prev_bf16  the previous step's output (same n), or NULL after the first
 *                step (no distance; only the step count advances)
 *   delta        threshold, finite and >= 0
 *   state        as for qs_gbs_reset; updates on one state must not overlap
 */
QS_API qs_status qs_gbs_update(const void* y_cur_bf16, const void* y_prev_bf16, int64_t n,
                               double delta, void* state, void* stream);

/*
 * qs_linear_gbs — the one-call layer (as qs_linear) at the width the state
 * holds: the 4-bit and the 8-bit kernels are both enqueued and each returns at
 * once unless the state selects its width.  Weights are prepared at both
 * widths: qs_pack_weights with bits 8, and with bits 4 and QS_FLAG_BYTE_CODES
 * (the 4-bit codes one per byte, [N][K] bytes).  With both operands stored in
 * bytes the 4-bit step runs the 8-bit-storage GEMM on 4-bit codes: the int8
 * tensor cores multiply them no faster, and that GEMM, which runs at the
 * board's power limit, clocks higher on 4-bit values than the packed 4x4
 * GEMM runs in the same sequence.
 *   w4_packed, w4_scale  weights at 4 bits, one code per byte;
 *   w8_packed, w8_scale  weights at 8 bits
 *   state                a qs_gbs_state (read only)
 *   workspace            at least qs_linear_workspace_bytes(M, K, 8) bytes
 *   other arguments as qs_linear
 */
QS_API qs_status qs_linear_gbs(const void* x_bf16, int64_t M, int64_t K, float alpha,
                               const void* w4_packed, const float* w4_scale,
                               const void* w8_packed, const float* w8_scale,
                               const void* bias_bf16, int64_t N, const void* state,
                               void* workspace, int64_t workspace_bytes, void* out_bf16,
                               void* stream);

/*
 * qs_gelu_bf16 — elementwise GELU (exact erf form, binary32 arithmetic,
 * bf16 in and out) used between the ffn-up and ffn-down linears of a
 * transformer block chain.  n elements; x and y may alias (each element is
 * read and written by the same thread).  For n >= 2^24 each CTA first
 * tabulates the function over all 65536 bf16 inputs in shared memory and
 * then reads the table: the same bits as the direct evaluation.
 * Errors: QS_ERR_NULL, QS_ERR_SHAPE (n <= 0), QS_ERR_ALIGN (x or y not
 * 16-byte aligned), QS_ERR_PTR (not device memory of the current device),
 * QS_ERR_CUDA.
 */
QS_API qs_status qs_gelu_bf16(const void* x_bf16, int64_t n, void* y_bf16, void* stream);

/*
 * qs_linear_noalloc — qs_linear for callers that cannot allocate device memory
 * when they run the layer: a host runtime that owns the whole device memory
 * pool and forbids other allocations, a plugin interface that hands over only
 * inputs and outputs with no workspace, or a latency-critical loop that cannot
 * afford an allocation (and the synchronisation cudaMalloc implies) per call.
 * The scratch qs_linear would take from the caller comes instead from a
 * buffer of QS_NOALLOC_SCRATCH_BYTES that the library keeps in device memory
 * (every GPU that loads libqs.so holds it until the process exits).  Nothing
 * is allocated by this call.
 *   Arguments as qs_linear, minus the workspace.  Calls needing more scratch
 *   than the buffer, i.e. qs_linear_workspace_bytes(M, K, bits) >
 *   QS_NOALLOC_SCRATCH_BYTES, are rejected with QS_ERR_RANGE (W4, K = 5120:
 *   up to 3271 tokens per call).
 *   The first call on a device looks up the buffer's device address (with
 *   that device current); make that first call before any stream capture.
 *   The address is kept per device together with the id of the CUDA context
 *   it was taken in; a call from a different context (for instance after
 *   cudaDeviceReset, when the library's module may load elsewhere) looks it
 *   up again, so the first call after a reset should also come before any
 *   capture.
 *   All calls share the one buffer, which keeps the previous call's contents
 *   (every byte the layer reads from it is written earlier in the same call,
 *   so nothing needs clearing); calls that may overlap on the GPU -- on
 *   different streams, or from different host threads -- race on it.
 * The pages have no counterpart: this is a deployment variant of qs_linear.
 */
#define QS_NOALLOC_SCRATCH_BYTES (8u << 20)
QS_API qs_status qs_linear_noalloc(const void* x_bf16, int64_t M, int64_t K, float alpha,
                                   const void* w_packed, const float* w_scale,
                                   const void* bias_bf16, int64_t N, int bits, void* out_bf16,
                                   void* stream);

/*
 * qs_selftest_timeout — diagnostic of the failure path: enqueues one tiny
 * kernel whose bounded mbarrier wait can never complete (nothing arrives); the
 * wait gives up after `timeout_us` microseconds (1 .. 1000000), records the
 * timeout in the device error word and the kernel returns.  A following
 * qs_device_error() then reports QS_ERR_TIMEOUT and the context stays usable.
 * No counterpart on the pages.
 */
QS_API qs_status qs_selftest_timeout(int64_t timeout_us, void* stream);

/*
 * qs_device_error — synchronises `stream`, then returns and clears the
 * library's device-side error word: QS_OK, QS_ERR_TIMEOUT if a kernel gave up
 * a bounded wait (its outputs are then undefined), QS_ERR_RANGE if a row index
 * read on the device was out of range (and no wait gave up), or QS_ERR_CUDA if
 * the synchronisation itself failed.
 */
QS_API qs_status qs_device_error(void* stream);

/* Static description of a status code. */
QS_API const char* qs_status_str(int status);

/* Library version string. */
QS_API const char* qs_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QS_H_ */
