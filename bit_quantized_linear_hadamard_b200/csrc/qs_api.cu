// libqs.so — C ABI entry points: argument validation, tensor-map set-up and
// launches of the rotate-quantize kernel, the tcgen05 GEMM and the GELU glue.
// See include/qs.h for the contract of every function.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "qs.h"
#include "qs_bgr.cuh"
#include "qs_gbs.cuh"
#include "qs_gemm.cuh"
#include "qs_host.cuh"
#include "qs_glue.cuh"
#include "qs_quant.cuh"
#include "qs_sd4.cuh"
#include "qs_sd4_mx.cuh"

namespace {

using qs::gemm::dispatch_qgemm;
using qs::gemm::launch_qgemm;

constexpr unsigned kKnownFlags = QS_FLAG_NO_ROTATE | QS_FLAG_BYTE_CODES;
constexpr float kMinAlpha = 1.0f / 16384.0f;  // keeps |u * inv| < 2^22

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The pointer must be device (or managed) memory usable by the current device.
qs_status check_device_ptr(const void* p) {
  cudaPointerAttributes a;
  const cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return QS_ERR_PTR;
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return QS_ERR_PTR;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return QS_ERR_CUDA;
  if (a.type == cudaMemoryTypeDevice && a.device != dev) return QS_ERR_PTR;
  return QS_OK;
}

qs_status check_rows_k(int64_t rows, int64_t K) {
  if (rows <= 0 || K <= 0 || K % 128 != 0) return QS_ERR_SHAPE;
  if (K > QS_MAX_K || rows > QS_MAX_ROWS) return QS_ERR_RANGE;
  return QS_OK;
}

qs_status check_bits(int bits) {
  return (bits == 4 || bits == 6 || bits == 8) ? QS_OK : QS_ERR_BITS;
}

// Bytes of one packed row of K codes.
int64_t packed_row_bytes(int64_t K, int bits) { return K * qs::code_storage_bits(bits) / 8; }

#define QS_TRY(expr)               \
  do {                             \
    const qs_status _s = (expr);   \
    if (_s != QS_OK) return _s;    \
  } while (0)

qs_status check_gemm_args(const void* xp, const void* wp, const void* out, int64_t M, int64_t N,
                          int64_t K, int bits_x, int bits_w) {
  if (!xp || !wp || !out) return QS_ERR_NULL;
  QS_TRY(check_bits(bits_x));
  QS_TRY(check_bits(bits_w));
  QS_TRY(check_rows_k(M, K));
  QS_TRY(check_rows_k(N, K));
  if (N % 16 != 0) return QS_ERR_SHAPE;
  if (M > INT32_MAX || N > INT32_MAX) return QS_ERR_RANGE;
  if (!aligned16(xp) || !aligned16(wp) || !aligned16(out)) return QS_ERR_ALIGN;
  return QS_OK;
}

// Scratch of qs_linear_noalloc: one fixed buffer per device, in the module's
// global memory (no allocation).  Host code only names the symbol; its device
// address is looked up once per device and context.
static __device__ __align__(256) unsigned char g_noalloc_scratch[QS_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mutex;
void* g_noalloc_addr[64] = {nullptr};
unsigned long long g_noalloc_ctx[64] = {0};  // context id the address belongs to

// Unique id of the calling thread's current CUDA context (driver entry points,
// no link-time libcuda dependency); 0 if it cannot be read.  A context created
// after cudaDeviceReset gets a new id even if it reuses the old handle's memory.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_noalloc_scratch on the current device, or nullptr if the
// lookup failed.  It is looked up with that device current on the first call
// for the device, and again whenever the calling thread's context differs from
// the one the cached address was taken in (after a cudaDeviceReset the module
// may load at another address), or cannot be identified.
void* noalloc_scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_addr[dev] && ctx != 0 && g_noalloc_ctx[dev] == ctx) return g_noalloc_addr[dev];
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  // the lookup has made the device's context current if it was not
  g_noalloc_addr[dev] = p;
  g_noalloc_ctx[dev] = current_context_id();
  return p;
}

// Persistent launch of the SD4 GEMM: one CTA per SM at most.
template <bool WDEC>
qs_status launch_sd4_gemm(const CUtensorMap& ca, const CUtensorMap& cb, const CUtensorMap& ma,
                          const CUtensorMap& mb, const CUtensorMap& wb, const void* bias,
                          int64_t M, int64_t N, int64_t K, void* out, void* stream,
                          int64_t kb_wrap = 0, const int32_t* out_rows = nullptr,
                          int64_t out_M = 0) {
  namespace G = qs::sd4::gemm_sd4;
  constexpr int smem = G::SCfg<WDEC>::kSmemBytes;
  auto kern = G::sd4_gemm_kernel<WDEC>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return QS_ERR_CUDA;
  const int sms = qs::sm_count();
  if (sms <= 0) return QS_ERR_CUDA;
  const int64_t tiles = ((M + G::BM - 1) / G::BM) * ((N + G::BN - 1) / G::BN);
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  kern<<<grid, G::kThreads, smem, static_cast<cudaStream_t>(stream)>>>(
      ca, cb, ma, mb, wb, static_cast<const uint16_t*>(bias), static_cast<uint16_t*>(out),
      static_cast<int>(M), static_cast<int>(N), static_cast<int>(K),
      static_cast<int>(kb_wrap > 0 ? kb_wrap : K / G::BK), out_rows,
      static_cast<int>(out_rows ? out_M : M));
  return cudaGetLastError() == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}

template <bool ADEC, bool BDEC, bool WIDE = false, bool TILES = false>
qs_status launch_sd4_mx(const CUtensorMap& ca, const CUtensorMap& cb, const CUtensorMap& ma,
                        const CUtensorMap& mb, const CUtensorMap& xa, const CUtensorMap& wb,
                        const void* bias, int64_t M, int64_t N, int64_t K, void* out,
                        void* stream, int64_t kb_wrap, const int32_t* out_rows, int64_t out_M,
                        const void* a_tiles = nullptr, const void* b_tiles = nullptr) {
  namespace G = qs::sd4::gemm_mx;
  using C = G::MCfg<ADEC, BDEC, WIDE, TILES>;
  constexpr int smem = C::kSmemBytes;
  auto kern = G::sd4_mx_gemm_kernel<ADEC, BDEC, WIDE, TILES>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return QS_ERR_CUDA;
  const int sms = qs::sm_count();
  if (sms <= 0) return QS_ERR_CUDA;
  const int64_t tiles = ((M + G::BM - 1) / G::BM) * ((N + C::kBN - 1) / C::kBN);
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  kern<<<grid, C::kThreads, smem, static_cast<cudaStream_t>(stream)>>>(
      ca, cb, ma, mb, xa, wb, static_cast<const uint16_t*>(bias), static_cast<uint16_t*>(out),
      static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), static_cast<int>(kb_wrap),
      out_rows, static_cast<int>(out_rows ? out_M : M), static_cast<const uint8_t*>(a_tiles),
      static_cast<const uint8_t*>(b_tiles));
  return cudaGetLastError() == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}

// The block-scaled SD4 GEMM: A = `a_rows` rows of Ka elements (Ka = K, or 2K
// for decomposed rows) as codes or, when a_e4m3 is not NULL, as e4m3 bytes;
// the weights as codes or, when w_e4m3 is not NULL, as e4m3 bytes; block
// words for both.
qs_status run_sd4_mx(const void* a_codes, const void* a_e4m3, const uint16_t* a_meta,
                     int64_t a_rows, int64_t Ka, const void* w_codes, const void* w_e4m3,
                     const uint16_t* w_meta, const void* bias, int64_t N, int64_t K, void* out,
                     void* stream, const int32_t* out_rows, int64_t out_M) {
  namespace G = qs::sd4::gemm_mx;
  CUtensorMap ca, ma, cb, mb, xa, wb;
  if (!qs::make_tensor_map_2d(&ma, a_meta, static_cast<uint64_t>(Ka) / 16,
                              static_cast<uint64_t>(a_rows), 16, G::BM, false) ||
      !qs::make_tensor_map_2d(&mb, w_meta, static_cast<uint64_t>(K) / 16,
                              static_cast<uint64_t>(N), 16, G::BN, false))
    return QS_ERR_CUDA;
  if (a_e4m3 ? !qs::make_tensor_map_2d(&xa, a_e4m3, static_cast<uint64_t>(Ka),
                                       static_cast<uint64_t>(a_rows), G::BK, G::BM, true)
             : !qs::make_tensor_map_2d(&ca, a_codes, static_cast<uint64_t>(Ka) / 2,
                                       static_cast<uint64_t>(a_rows), G::BK / 2, G::BM, false))
    return QS_ERR_CUDA;
  if (w_e4m3 ? !qs::make_tensor_map_2d(&wb, w_e4m3, static_cast<uint64_t>(K),
                                       static_cast<uint64_t>(N), G::BK, G::BN, true)
             : !qs::make_tensor_map_2d(&cb, w_codes, static_cast<uint64_t>(K) / 2,
                                       static_cast<uint64_t>(N), G::BK / 2, G::BN, false))
    return QS_ERR_CUDA;
  const int64_t kb_wrap = K / G::BK;
  if (a_e4m3) {
    if (!w_e4m3) return QS_ERR_NULL;  // e4m3 activations go with e4m3 weights
    return launch_sd4_mx<false, false, true>(xa, xa, ma, mb, xa, wb, bias, a_rows, N, Ka, out,
                                             stream, kb_wrap, out_rows, out_M);
  }
  if (w_e4m3)
    return launch_sd4_mx<true, false>(ca, ca, ma, mb, ca, wb, bias, a_rows, N, Ka, out, stream,
                                      kb_wrap, out_rows, out_M);
  return launch_sd4_mx<true, true>(ca, cb, ma, mb, ca, cb, bias, a_rows, N, Ka, out, stream,
                                   kb_wrap, out_rows, out_M);
}

// The SD4 quantiser (dialect choice on the tensor cores): codes or e4m3 bytes.
template <bool E4M3>
qs_status launch_sd4_quant_tc(const void* x, int64_t rows, int64_t K, void* out, uint16_t* meta,
                              void* stream) {
  namespace T = qs::sd4::tc;
  auto kern = T::sd4_quant_tc_kernel<E4M3>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, T::kSmemBytes) !=
      cudaSuccess)
    return QS_ERR_CUDA;
  const int sms = qs::sm_count();
  if (sms <= 0) return QS_ERR_CUDA;
  const int64_t tiles = (rows * (K / 32) + T::kTileBlocks - 1) / T::kTileBlocks;
  int64_t grid = static_cast<int64_t>(sms) * 4;  // four CTAs fit an SM's shared memory
  if (grid > tiles) grid = tiles;
  kern<<<static_cast<unsigned>(grid), T::kThreads, T::kSmemBytes,
         static_cast<cudaStream_t>(stream)>>>(static_cast<const uint16_t*>(x), rows,
                                              static_cast<int>(K), static_cast<uint8_t*>(out), meta);
  return cudaGetLastError() == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}

}  // namespace

extern "C" {

qs_status qs_pack_weights(const void* w_bf16, int64_t N, int64_t K, int bits, unsigned flags,
                          void* w_packed, float* w_scale, void* stream) {
  if (!w_bf16 || !w_packed || !w_scale) return QS_ERR_NULL;
  QS_TRY(check_bits(bits));
  QS_TRY(check_rows_k(N, K));
  if (flags & ~kKnownFlags) return QS_ERR_RANGE;
  if (!aligned16(w_bf16) || !aligned16(w_packed) || !aligned16(w_scale)) return QS_ERR_ALIGN;
  QS_TRY(check_device_ptr(w_bf16));
  QS_TRY(check_device_ptr(w_packed));
  QS_TRY(check_device_ptr(w_scale));
  const bool rotate = !(flags & QS_FLAG_NO_ROTATE);
  // (1/sqrt(128))^2 of the two rotations, exact in binary32.
  const float scale_mul = rotate ? 0.0078125f : 1.0f;
  const cudaError_t e = qs::launch_rotate_quant(
      static_cast<const uint16_t*>(w_bf16), N, static_cast<int>(K), bits, 1.0f, scale_mul,
      rotate ? 1 : 0, static_cast<uint8_t*>(w_packed), w_scale, static_cast<cudaStream_t>(stream),
      nullptr, 0, nullptr, (flags & QS_FLAG_BYTE_CODES) != 0);
  return e == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}

qs_status qs_quant_act(const void* x_bf16, int64_t M, int64_t K, int bits, float alpha,
                       unsigned flags, void* x_packed, float* x_scale, void* stream) {
  if (!x_bf16 || !x_packed || !x_scale) return QS_ERR_NULL;
  QS_TRY(check_bits(bits));
  QS_TRY(check_rows_k(M, K));
  if (!(alpha >= kMinAlpha && alpha <= 1.0f)) return QS_ERR_RANGE;
  if (flags & ~kKnownFlags) return QS_ERR_RANGE;
  if (!aligned16(x_bf16) || !aligned16(x_packed) || !aligned16(x_scale)) return QS_ERR_ALIGN;
  QS_TRY(check_device_ptr(x_bf16));
  QS_TRY(check_device_ptr(x_packed));
  QS_TRY(check_device_ptr(x_scale));
  const bool rotate = !(flags & QS_FLAG_NO_ROTATE);
  const cudaError_t e = qs::launch_rotate_quant(
      static_cast<const uint16_t*>(x_bf16), M, static_cast<int>(K), bits, alpha, 1.0f,
      rotate ? 1 : 0, static_cast<uint8_t*>(x_packed), x_scale, static_cast<cudaStream_t>(stream),
      nullptr, 0, nullptr, (flags & QS_FLAG_BYTE_CODES) != 0);
  return e == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}

qs_status qs_qlinear_mixed(const void* x_packed, const float* x_scale, int bits_x,
                           const void* w_packed, const float* w_scale, int bits_w,
                           const void* bias_bf16, int64_t M, int64_t N, int64_t K,
                           void* out_bf16, void* stream) {
  QS_TRY(check_gemm_args(x_packed, w_packed, out_bf16, M, N, K, bits_x, bits_w));
  if (!x_scale || !w_scale) return QS_ERR_NULL;
  if (!aligned16(x_scale) || !aligned16(w_scale) || (bias_bf16 && !aligned16(bias_bf16)))
    return QS_ERR_ALIGN;
  QS_TRY(check_device_ptr(x_packed));
  QS_TRY(check_device_ptr(w_packed));
  QS_TRY(check_device_ptr(x_scale));
  QS_TRY(check_device_ptr(w_scale));
  QS_TRY(check_device_ptr(out_bf16));
  if (bias_bf16) QS_TRY(check_device_ptr(bias_bf16));
  return dispatch_qgemm<false>(bits_x, bits_w, x_packed, x_scale, w_packed, w_scale, bias_bf16, M,
                               N, K, out_bf16, static_cast<cudaStream_t>(stream));
}

qs_status qs_qlinear(const void* x_packed, const float* x_scale, const void* w_packed,
                     const float* w_scale, const void* bias_bf16, int64_t M, int64_t N,
                     int64_t K, int bits, void* out_bf16, void* stream) {
  return qs_qlinear_mixed(x_packed, x_scale, bits, w_packed, w_scale, bits, bias_bf16, M, N, K,
                          out_bf16, stream);
}

qs_status qs_qgemm_s32_mixed(const void* x_packed, int bits_x, const void* w_packed, int bits_w,
                             int64_t M, int64_t N, int64_t K, int32_t* acc, void* stream) {
  QS_TRY(check_gemm_args(x_packed, w_packed, acc, M, N, K, bits_x, bits_w));
  QS_TRY(check_device_ptr(x_packed));
  QS_TRY(check_device_ptr(w_packed));
  QS_TRY(check_device_ptr(acc));
  return dispatch_qgemm<true>(bits_x, bits_w, x_packed, nullptr, w_packed, nullptr, nullptr, M, N,
                              K, acc, static_cast<cudaStream_t>(stream));
}

qs_status qs_qgemm_s32(const void* x_packed, const void* w_packed, int64_t M, int64_t N,
                       int64_t K, int bits, int32_t* acc, void* stream) {
  return qs_qgemm_s32_mixed(x_packed, bits, w_packed, bits, M, N, K, acc, stream);
}

int64_t qs_linear_workspace_bytes(int64_t M, int64_t K, int bits) {
  if (check_bits(bits) != QS_OK || check_rows_k(M, K) != QS_OK) return -1;
  const int64_t packed = (M * packed_row_bytes(K, bits) + 255) / 256 * 256;
  return packed + 4 * M;
}

qs_status qs_linear_ex(const void* x_bf16, int64_t M, int64_t K, float alpha, int bits_x,
                       unsigned x_flags, const void* w_packed, const float* w_scale, int bits_w,
                       const void* bias_bf16, int64_t N, void* workspace, int64_t workspace_bytes,
                       void* out_bf16, void* stream) {
  if (!x_bf16 || !w_packed || !w_scale || !workspace || !out_bf16) return QS_ERR_NULL;
  QS_TRY(check_gemm_args(workspace, w_packed, out_bf16, M, N, K, bits_x, bits_w));
  if (!(alpha >= kMinAlpha && alpha <= 1.0f)) return QS_ERR_RANGE;
  if (x_flags & ~kKnownFlags) return QS_ERR_RANGE;
  // storage width of the activation codes, which is what the GEMM reads
  const int store_x = (x_flags & QS_FLAG_BYTE_CODES) ? 8 : bits_x;
  const int64_t need = qs_linear_workspace_bytes(M, K, store_x);
  if (need < 0) return QS_ERR_SHAPE;
  if (workspace_bytes < need) return QS_ERR_RANGE;
  // everything both launches will check, before the first one
  if (!aligned16(x_bf16) || !aligned16(w_scale) || (bias_bf16 && !aligned16(bias_bf16)))
    return QS_ERR_ALIGN;
  QS_TRY(check_device_ptr(x_bf16));
  QS_TRY(check_device_ptr(w_packed));
  QS_TRY(check_device_ptr(w_scale));
  QS_TRY(check_device_ptr(workspace));
  QS_TRY(check_device_ptr(out_bf16));
  if (bias_bf16) QS_TRY(check_device_ptr(bias_bf16));
  uint8_t* xp = static_cast<uint8_t*>(workspace);
  float* xs = reinterpret_cast<float*>(xp + (M * packed_row_bytes(K, store_x) + 255) / 256 * 256);
  QS_TRY(qs_quant_act(x_bf16, M, K, bits_x, alpha, x_flags, xp, xs, stream));
  return qs_qlinear_mixed(xp, xs, store_x, w_packed, w_scale, bits_w, bias_bf16, M, N, K,
                          out_bf16, stream);
}

qs_status qs_linear_mixed(const void* x_bf16, int64_t M, int64_t K, float alpha, int bits_x,
                          const void* w_packed, const float* w_scale, int bits_w,
                          const void* bias_bf16, int64_t N, void* workspace,
                          int64_t workspace_bytes, void* out_bf16, void* stream) {
  return qs_linear_ex(x_bf16, M, K, alpha, bits_x, 0u, w_packed, w_scale, bits_w, bias_bf16, N,
                      workspace, workspace_bytes, out_bf16, stream);
}

qs_status qs_linear(const void* x_bf16, int64_t M, int64_t K, float alpha, const void* w_packed,
                    const float* w_scale, const void* bias_bf16, int64_t N, int bits,
                    void* workspace, int64_t workspace_bytes, void* out_bf16, void* stream) {
  return qs_linear_mixed(x_bf16, M, K, alpha, bits, w_packed, w_scale, bits, bias_bf16, N,
                         workspace, workspace_bytes, out_bf16, stream);
}

qs_status qs_gbs_reset(void* state, void* stream) {
  if (!state) return QS_ERR_NULL;
  if (!aligned16(state)) return QS_ERR_ALIGN;
  QS_TRY(check_device_ptr(state));
  qs::gbs::gbs_reset_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<qs_gbs_state*>(state));
  return cudaGetLastError() == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}

qs_status qs_gbs_update(const void* y_cur_bf16, const void* y_prev_bf16, int64_t n, double delta,
                        void* state, void* stream) {
  if (!y_cur_bf16 || !state) return QS_ERR_NULL;
  if (n <= 0) return QS_ERR_SHAPE;
  if (!(delta >= 0.0 && delta <= 1.7976931348623157e308)) return QS_ERR_RANGE;
  if (!aligned16(y_cur_bf16) || !aligned16(state) || (y_prev_bf16 && !aligned16(y_prev_bf16)))
    return QS_ERR_ALIGN;
  QS_TRY(check_device_ptr(y_cur_bf16));
  QS_TRY(check_device_ptr(state));
  if (y_prev_bf16) QS_TRY(check_device_ptr(y_prev_bf16));
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  qs_gbs_state* st = static_cast<qs_gbs_state*>(state);
  if (!y_prev_bf16) {
    qs::gbs::gbs_first_kernel<<<1, 1, 0, s>>>(delta, st);
    return cudaGetLastError() == cudaSuccess ? QS_OK : QS_ERR_CUDA;
  }
  const int sms = qs::sm_count();
  if (sms <= 0) return QS_ERR_CUDA;
  // a fixed grid per device and size keeps the summation order fixed
  const int64_t nvec = n / 8;
  int64_t blocks = (nvec + qs::gbs::kThreads - 1) / qs::gbs::kThreads;
  const int64_t cap = static_cast<int64_t>(sms) * 4 < qs::gbs::kMaxBlocks
                          ? static_cast<int64_t>(sms) * 4
                          : qs::gbs::kMaxBlocks;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  qs::gbs::gbs_update_kernel<<<static_cast<unsigned>(blocks), qs::gbs::kThreads, 0, s>>>(
      static_cast<const uint16_t*>(y_cur_bf16), static_cast<const uint16_t*>(y_prev_bf16), n,
      delta, st);
  return cudaGetLastError() == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}

qs_status qs_linear_gbs(const void* x_bf16, int64_t M, int64_t K, float alpha,
                        const void* w4_packed, const float* w4_scale, const void* w8_packed,
                        const float* w8_scale, const void* bias_bf16, int64_t N,
                        const void* state, void* workspace, int64_t workspace_bytes,
                        void* out_bf16, void* stream) {
  if (!x_bf16 || !w4_packed || !w4_scale || !w8_packed || !w8_scale || !state || !workspace ||
      !out_bf16)
    return QS_ERR_NULL;
  QS_TRY(check_gemm_args(workspace, w4_packed, out_bf16, M, N, K, 4, 4));
  QS_TRY(check_gemm_args(workspace, w8_packed, out_bf16, M, N, K, 8, 8));
  if (!(alpha >= kMinAlpha && alpha <= 1.0f)) return QS_ERR_RANGE;
  const int64_t need = qs_linear_workspace_bytes(M, K, 8);
  if (need < 0) return QS_ERR_SHAPE;
  if (workspace_bytes < need) return QS_ERR_RANGE;
  if (!aligned16(x_bf16) || !aligned16(w4_scale) || !aligned16(w8_scale) || !aligned16(state) ||
      (bias_bf16 && !aligned16(bias_bf16)))
    return QS_ERR_ALIGN;
  for (const void* p : {x_bf16, w4_packed, static_cast<const void*>(w4_scale), w8_packed,
                        static_cast<const void*>(w8_scale), state,
                        static_cast<const void*>(workspace), static_cast<const void*>(out_bf16)})
    QS_TRY(check_device_ptr(p));
  if (bias_bf16) QS_TRY(check_device_ptr(bias_bf16));
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the width word of the state, read by every gated kernel when it starts
  const int* gate = &static_cast<const qs_gbs_state*>(state)->bits;
  uint8_t* xp = static_cast<uint8_t*>(workspace);
  float* xs = reinterpret_cast<float*>(xp + (M * K + 255) / 256 * 256);
  const uint16_t* x = static_cast<const uint16_t*>(x_bf16);
  // The 4-bit step stores its activation codes one per byte and takes the
  // 4-bit weight codes one per byte as well, so it runs the 8-bit-storage GEMM
  // on 4-bit values.  The int8 tensor cores multiply 4-bit codes no faster
  // than 8-bit ones, and that GEMM runs at the board's power limit, where
  // 4-bit values (fewer toggling bits) let it clock higher: inside the step
  // sequence this form took 1.41-1.42 ms per layer call against 1.49-1.50 ms
  // for the packed 4x4 GEMM, and 1.53 ms for the 8-bit step.
  for (int bits : {4, 8})
    if (qs::launch_rotate_quant(x, M, static_cast<int>(K), bits, alpha, 1.0f, 1, xp, xs, s, gate,
                                bits, nullptr, /*byte_codes=*/true) != cudaSuccess)
      return QS_ERR_CUDA;
  const qs_status st4 = launch_qgemm<8, 8, false>(xp, xs, w4_packed, w4_scale, bias_bf16, M, N, K,
                                                  out_bf16, s, gate, 4);
  if (st4 != QS_OK) return st4;
  return launch_qgemm<8, 8, false>(xp, xs, w8_packed, w8_scale, bias_bf16, M, N, K, out_bf16, s,
                                   gate, 8);
}

qs_status qs_pack_weights_bgr(const void* w_bf16, int64_t N, int64_t K, int bits, unsigned flags,
                              int candidates, int iterations, void* w_packed, float* w_scale,
                              int32_t* w_offset, void* stream) {
  if (!w_bf16 || !w_packed || !w_scale || !w_offset) return QS_ERR_NULL;
  if (bits != 4 && bits != 8) return QS_ERR_BITS;
  QS_TRY(check_rows_k(N, K));
  if (K > qs::bgr::kMaxK || candidates < 1 || candidates > qs::bgr::kMaxCandidates ||
      iterations < 0 || iterations > 64 || (flags & ~kKnownFlags))
    return QS_ERR_RANGE;
  if (N > INT32_MAX) return QS_ERR_RANGE;
  if (!aligned16(w_bf16) || !aligned16(w_packed) || !aligned16(w_scale) || !aligned16(w_offset))
    return QS_ERR_ALIGN;
  QS_TRY(check_device_ptr(w_bf16));
  QS_TRY(check_device_ptr(w_packed));
  QS_TRY(check_device_ptr(w_scale));
  QS_TRY(check_device_ptr(w_offset));
  const bool rotate = !(flags & QS_FLAG_NO_ROTATE);
  const int smem = static_cast<int>(K) * 4;
  auto kern = bits == 4 ? qs::bgr::bgr_pack_kernel<4> : qs::bgr::bgr_pack_kernel<8>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return QS_ERR_CUDA;
  kern<<<static_cast<unsigned>(N), qs::bgr::kThreads, smem, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(w_bf16), static_cast<int>(K), rotate ? 1 : 0, candidates,
      iterations, rotate ? 0.0078125f : 1.0f, static_cast<uint8_t*>(w_packed), w_scale, w_offset);
  return cudaGetLastError() == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}

qs_status qs_quant_act_rowsum(const void* x_bf16, int64_t M, int64_t K, int bits, float alpha,
                              unsigned flags, void* x_packed, float* x_scale, int32_t* x_rowsum,
                              void* stream) {
  if (!x_rowsum) return QS_ERR_NULL;
  if (!aligned16(x_rowsum)) return QS_ERR_ALIGN;
  if (!x_bf16 || !x_packed || !x_scale) return QS_ERR_NULL;
  QS_TRY(check_bits(bits));
  QS_TRY(check_rows_k(M, K));
  if (!(alpha >= kMinAlpha && alpha <= 1.0f)) return QS_ERR_RANGE;
  if (flags & ~kKnownFlags) return QS_ERR_RANGE;
  if (!aligned16(x_bf16) || !aligned16(x_packed) || !aligned16(x_scale)) return QS_ERR_ALIGN;
  for (const void* p : {x_bf16, static_cast<const void*>(x_packed),
                        static_cast<const void*>(x_scale), static_cast<const void*>(x_rowsum)})
    QS_TRY(check_device_ptr(p));
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(x_rowsum, 0, static_cast<size_t>(M) * 4, s) != cudaSuccess)
    return QS_ERR_CUDA;
  const bool rotate = !(flags & QS_FLAG_NO_ROTATE);
  const cudaError_t e = qs::launch_rotate_quant(
      static_cast<const uint16_t*>(x_bf16), M, static_cast<int>(K), bits, alpha, 1.0f,
      rotate ? 1 : 0, static_cast<uint8_t*>(x_packed), x_scale, s, nullptr, 0, x_rowsum,
      (flags & QS_FLAG_BYTE_CODES) != 0);
  return e == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}

qs_status qs_qlinear_asym(const void* x_packed, const float* x_scale, const int32_t* x_rowsum,
                          const void* w_packed, const float* w_scale, const int32_t* w_offset,
                          const void* bias_bf16, int64_t M, int64_t N, int64_t K, int bits,
                          void* out_bf16, void* stream) {
  if (bits != 4 && bits != 8) return QS_ERR_BITS;
  QS_TRY(check_gemm_args(x_packed, w_packed, out_bf16, M, N, K, bits, bits));
  if (!x_scale || !w_scale || !x_rowsum || !w_offset) return QS_ERR_NULL;
  if (!aligned16(x_scale) || !aligned16(w_scale) || !aligned16(x_rowsum) ||
      !aligned16(w_offset) || (bias_bf16 && !aligned16(bias_bf16)))
    return QS_ERR_ALIGN;
  for (const void* p : {x_packed, static_cast<const void*>(x_scale),
                        static_cast<const void*>(x_rowsum), w_packed,
                        static_cast<const void*>(w_scale), static_cast<const void*>(w_offset),
                        static_cast<const void*>(out_bf16)})
    QS_TRY(check_device_ptr(p));
  if (bias_bf16) QS_TRY(check_device_ptr(bias_bf16));
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  return bits == 4 ? launch_qgemm<4, 4, false, true>(x_packed, x_scale, w_packed, w_scale,
                                                      bias_bf16, M, N, K, out_bf16, s, nullptr, 0,
                                                      x_rowsum, w_offset)
                   : launch_qgemm<8, 8, false, true>(x_packed, x_scale, w_packed, w_scale,
                                                      bias_bf16, M, N, K, out_bf16, s, nullptr, 0,
                                                      x_rowsum, w_offset);
}

qs_status qs_qgemm_s32_asym(const void* x_packed, const int32_t* x_rowsum, const void* w_packed,
                            const int32_t* w_offset, int64_t M, int64_t N, int64_t K, int bits,
                            int32_t* acc, void* stream) {
  if (bits != 4 && bits != 8) return QS_ERR_BITS;
  QS_TRY(check_gemm_args(x_packed, w_packed, acc, M, N, K, bits, bits));
  if (!x_rowsum || !w_offset) return QS_ERR_NULL;
  if (!aligned16(x_rowsum) || !aligned16(w_offset)) return QS_ERR_ALIGN;
  for (const void* p : {x_packed, static_cast<const void*>(x_rowsum), w_packed,
                        static_cast<const void*>(w_offset), static_cast<const void*>(acc)})
    QS_TRY(check_device_ptr(p));
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  return bits == 4 ? launch_qgemm<4, 4, true, true>(x_packed, nullptr, w_packed, nullptr, nullptr,
                                                     M, N, K, acc, s, nullptr, 0, x_rowsum,
                                                     w_offset)
                   : launch_qgemm<8, 8, true, true>(x_packed, nullptr, w_packed, nullptr, nullptr,
                                                     M, N, K, acc, s, nullptr, 0, x_rowsum,
                                                     w_offset);
}

int64_t qs_linear_bgr_workspace_bytes(int64_t M, int64_t K, int bits) {
  if ((bits != 4 && bits != 8) || check_rows_k(M, K) != QS_OK) return -1;
  return (M * packed_row_bytes(K, bits) + 255) / 256 * 256 + (4 * M + 255) / 256 * 256 + 4 * M;
}

qs_status qs_linear_bgr(const void* x_bf16, int64_t M, int64_t K, float alpha,
                        const void* w_packed, const float* w_scale, const int32_t* w_offset,
                        const void* bias_bf16, int64_t N, int bits, void* workspace,
                        int64_t workspace_bytes, void* out_bf16, void* stream) {
  if (!x_bf16 || !w_packed || !w_scale || !w_offset || !workspace || !out_bf16)
    return QS_ERR_NULL;
  if (bits != 4 && bits != 8) return QS_ERR_BITS;
  QS_TRY(check_gemm_args(workspace, w_packed, out_bf16, M, N, K, bits, bits));
  if (!(alpha >= kMinAlpha && alpha <= 1.0f)) return QS_ERR_RANGE;
  const int64_t need = qs_linear_bgr_workspace_bytes(M, K, bits);
  if (need < 0) return QS_ERR_SHAPE;
  if (workspace_bytes < need) return QS_ERR_RANGE;
  if (!aligned16(x_bf16) || !aligned16(w_scale) || !aligned16(w_offset) ||
      (bias_bf16 && !aligned16(bias_bf16)))
    return QS_ERR_ALIGN;
  for (const void* p : {x_bf16, w_packed, static_cast<const void*>(w_scale),
                        static_cast<const void*>(w_offset), static_cast<const void*>(workspace),
                        static_cast<const void*>(out_bf16)})
    QS_TRY(check_device_ptr(p));
  if (bias_bf16) QS_TRY(check_device_ptr(bias_bf16));
  uint8_t* xp = static_cast<uint8_t*>(workspace);
  float* xs = reinterpret_cast<float*>(xp + (M * packed_row_bytes(K, bits) + 255) / 256 * 256);
  int32_t* xr = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(xs) + (4 * M + 255) / 256 * 256);
  QS_TRY(qs_quant_act_rowsum(x_bf16, M, K, bits, alpha, 0u, xp, xs, xr, stream));
  return qs_qlinear_asym(xp, xs, xr, w_packed, w_scale, w_offset, bias_bf16, M, N, K, bits,
                         out_bf16, stream);
}

qs_status qs_sd4_quant(const void* x_bf16, int64_t rows, int64_t K, void* codes, uint16_t* meta,
                       void* stream) {
  if (!x_bf16 || !codes || !meta) return QS_ERR_NULL;
  if (rows <= 0 || K <= 0 || K % 256 != 0) return QS_ERR_SHAPE;
  if (K > QS_MAX_K || rows > QS_MAX_ROWS) return QS_ERR_RANGE;
  if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(meta)) return QS_ERR_ALIGN;
  QS_TRY(check_device_ptr(x_bf16));
  QS_TRY(check_device_ptr(codes));
  QS_TRY(check_device_ptr(meta));
  return launch_sd4_quant_tc<false>(x_bf16, rows, K, codes, meta, stream);
}

qs_status qs_sd4_quant_e4m3(const void* x_bf16, int64_t rows, int64_t K, void* out_e4m3,
                            uint16_t* meta, void* stream) {
  if (!x_bf16 || !out_e4m3 || !meta) return QS_ERR_NULL;
  if (rows <= 0 || K <= 0 || K % 256 != 0) return QS_ERR_SHAPE;
  if (K > QS_MAX_K || rows > QS_MAX_ROWS) return QS_ERR_RANGE;
  if (!aligned16(x_bf16) || !aligned16(out_e4m3) || !aligned16(meta)) return QS_ERR_ALIGN;
  QS_TRY(check_device_ptr(x_bf16));
  QS_TRY(check_device_ptr(out_e4m3));
  QS_TRY(check_device_ptr(meta));
  return launch_sd4_quant_tc<true>(x_bf16, rows, K, out_e4m3, meta, stream);
}

qs_status qs_sd4_linear(const void* x_codes, const uint16_t* x_meta, const void* w_codes,
                        const uint16_t* w_meta, const void* bias_bf16, int64_t M, int64_t N,
                        int64_t K, void* out_bf16, void* stream) {
  if (!x_codes || !x_meta || !w_codes || !w_meta || !out_bf16) return QS_ERR_NULL;
  if (M <= 0 || N <= 0 || K <= 0 || K % 256 != 0 || N % 16 != 0) return QS_ERR_SHAPE;
  if (K > QS_MAX_K || M > INT32_MAX || N > INT32_MAX) return QS_ERR_RANGE;
  if (!aligned16(x_codes) || !aligned16(x_meta) || !aligned16(w_codes) || !aligned16(w_meta) ||
      !aligned16(out_bf16) || (bias_bf16 && !aligned16(bias_bf16)))
    return QS_ERR_ALIGN;
  for (const void* p : {x_codes, static_cast<const void*>(x_meta), w_codes,
                        static_cast<const void*>(w_meta), static_cast<const void*>(out_bf16)})
    QS_TRY(check_device_ptr(p));
  if (bias_bf16) QS_TRY(check_device_ptr(bias_bf16));
  return run_sd4_mx(x_codes, nullptr, x_meta, M, K, w_codes, nullptr, w_meta, bias_bf16, N, K,
                    out_bf16, stream, nullptr, 0);
}

qs_status qs_sd4_decode_e4m3(const void* codes, const uint16_t* meta, int64_t rows, int64_t K,
                             void* out_e4m3, void* stream) {
  if (!codes || !meta || !out_e4m3) return QS_ERR_NULL;
  if (rows <= 0 || K <= 0 || K % 256 != 0) return QS_ERR_SHAPE;
  if (K > QS_MAX_K || rows > QS_MAX_ROWS) return QS_ERR_RANGE;
  if (!aligned16(codes) || !aligned16(meta) || !aligned16(out_e4m3)) return QS_ERR_ALIGN;
  for (const void* p : {codes, static_cast<const void*>(meta), static_cast<const void*>(out_e4m3)})
    QS_TRY(check_device_ptr(p));
  const int sms = qs::sm_count();
  if (sms <= 0) return QS_ERR_CUDA;
  const int64_t tasks = rows * (K / 16);
  int64_t grid = (tasks + 255) / 256;
  if (grid > static_cast<int64_t>(sms) * 8) grid = static_cast<int64_t>(sms) * 8;
  qs::sd4::gemm_mx::sd4_decode_e4m3_kernel<<<static_cast<unsigned>(grid), 256, 0,
                                             static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(codes), meta, rows, static_cast<int>(K),
      static_cast<uint8_t*>(out_e4m3));
  return cudaGetLastError() == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}

qs_status qs_sd4_linear_e4m3w(const void* x_codes, const uint16_t* x_meta, const void* w_e4m3,
                              const uint16_t* w_meta, const void* bias_bf16, int64_t M, int64_t N,
                              int64_t K, void* out_bf16, void* stream) {
  if (!x_codes || !x_meta || !w_e4m3 || !w_meta || !out_bf16) return QS_ERR_NULL;
  if (M <= 0 || N <= 0 || K <= 0 || K % 256 != 0 || N % 16 != 0) return QS_ERR_SHAPE;
  if (K > QS_MAX_K || M > INT32_MAX || N > INT32_MAX) return QS_ERR_RANGE;
  if (!aligned16(x_codes) || !aligned16(x_meta) || !aligned16(w_e4m3) || !aligned16(w_meta) ||
      !aligned16(out_bf16) || (bias_bf16 && !aligned16(bias_bf16)))
    return QS_ERR_ALIGN;
  for (const void* p : {x_codes, static_cast<const void*>(x_meta), w_e4m3,
                        static_cast<const void*>(w_meta), static_cast<const void*>(out_bf16)})
    QS_TRY(check_device_ptr(p));
  if (bias_bf16) QS_TRY(check_device_ptr(bias_bf16));
  return run_sd4_mx(x_codes, nullptr, x_meta, M, K, nullptr, w_e4m3, w_meta, bias_bf16, N, K,
                    out_bf16, stream, nullptr, 0);
}

qs_status qs_sd4_linear_e4m3(const void* x_e4m3, const uint16_t* x_meta, const void* w_e4m3,
                             const uint16_t* w_meta, const void* bias_bf16, int64_t M, int64_t N,
                             int64_t K, void* out_bf16, void* stream) {
  if (!x_e4m3 || !x_meta || !w_e4m3 || !w_meta || !out_bf16) return QS_ERR_NULL;
  if (M <= 0 || N <= 0 || K <= 0 || K % 256 != 0 || N % 16 != 0) return QS_ERR_SHAPE;
  if (K > QS_MAX_K || M > INT32_MAX || N > INT32_MAX) return QS_ERR_RANGE;
  if (!aligned16(x_e4m3) || !aligned16(x_meta) || !aligned16(w_e4m3) || !aligned16(w_meta) ||
      !aligned16(out_bf16) || (bias_bf16 && !aligned16(bias_bf16)))
    return QS_ERR_ALIGN;
  for (const void* p : {x_e4m3, static_cast<const void*>(x_meta), w_e4m3,
                        static_cast<const void*>(w_meta), static_cast<const void*>(out_bf16)})
    QS_TRY(check_device_ptr(p));
  if (bias_bf16) QS_TRY(check_device_ptr(bias_bf16));
  return run_sd4_mx(nullptr, x_e4m3, x_meta, M, K, nullptr, w_e4m3, w_meta, bias_bf16, N, K,
                    out_bf16, stream, nullptr, 0);
}

int64_t qs_sd4_scale_tiles_bytes(int64_t rows, int64_t K, int weights) {
  namespace G = qs::sd4::gemm_mx;
  if (rows <= 0 || K <= 0 || K % 256 != 0 || K > QS_MAX_K || rows > QS_MAX_ROWS) return -1;
  const int64_t kbs = K / G::BK;
  if (weights) {  // groups of BN rows, whole 2-group tiles: 1024 bytes per group and stage
    const int64_t groups = 2 * ((rows + 2 * G::BN - 1) / (2 * G::BN));
    return groups * kbs * 2 * 512;
  }
  return ((rows + G::BM - 1) / G::BM) * kbs * 512;  // groups of BM rows
}

qs_status qs_sd4_scale_tiles(const uint16_t* meta, int64_t rows, int64_t K, int weights,
                             void* tiles, int64_t tiles_bytes, void* stream) {
  namespace G = qs::sd4::gemm_mx;
  if (!meta || !tiles) return QS_ERR_NULL;
  if (rows <= 0 || K <= 0 || K % 256 != 0) return QS_ERR_SHAPE;
  if (K > QS_MAX_K || rows > QS_MAX_ROWS || (weights != 0 && weights != 1)) return QS_ERR_RANGE;
  const int64_t need = qs_sd4_scale_tiles_bytes(rows, K, weights);
  if (tiles_bytes < need) return QS_ERR_RANGE;
  if (!aligned16(meta) || !aligned16(tiles)) return QS_ERR_ALIGN;
  QS_TRY(check_device_ptr(meta));
  QS_TRY(check_device_ptr(tiles));
  const int group = weights ? G::BN : G::BM;
  const int slots = weights ? 256 : 128;
  const int64_t groups = need / ((K / G::BK) * (slots / 128) * 512);
  const int sms = qs::sm_count();
  if (sms <= 0) return QS_ERR_CUDA;
  const int64_t tasks = groups * (K / G::BK) * slots;
  int64_t grid = (tasks + 255) / 256;
  if (grid > static_cast<int64_t>(sms) * 8) grid = static_cast<int64_t>(sms) * 8;
  G::sd4_scale_tiles_kernel<<<static_cast<unsigned>(grid), 256, 0,
                              static_cast<cudaStream_t>(stream)>>>(
      meta, rows, static_cast<int>(K), group, slots, groups, static_cast<uint8_t*>(tiles));
  return cudaGetLastError() == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}

qs_status qs_sd4_linear_e4m3_tiles(const void* x_e4m3, const void* x_tiles, const void* w_e4m3,
                                   const void* w_tiles, const void* bias_bf16, int64_t M,
                                   int64_t N, int64_t K, void* out_bf16, void* stream) {
  namespace G = qs::sd4::gemm_mx;
  if (!x_e4m3 || !x_tiles || !w_e4m3 || !w_tiles || !out_bf16) return QS_ERR_NULL;
  if (M <= 0 || N <= 0 || K <= 0 || K % 256 != 0 || N % 16 != 0) return QS_ERR_SHAPE;
  if (K > QS_MAX_K || M > INT32_MAX || N > INT32_MAX) return QS_ERR_RANGE;
  if (!aligned16(x_e4m3) || !aligned16(x_tiles) || !aligned16(w_e4m3) || !aligned16(w_tiles) ||
      !aligned16(out_bf16) || (bias_bf16 && !aligned16(bias_bf16)))
    return QS_ERR_ALIGN;
  for (const void* p : {x_e4m3, x_tiles, w_e4m3, w_tiles, static_cast<const void*>(out_bf16)})
    QS_TRY(check_device_ptr(p));
  if (bias_bf16) QS_TRY(check_device_ptr(bias_bf16));
  CUtensorMap xa, wb;
  if (!qs::make_tensor_map_2d(&xa, x_e4m3, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                              G::BK, G::BM, true) ||
      !qs::make_tensor_map_2d(&wb, w_e4m3, static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                              G::BK, G::BN, true))
    return QS_ERR_CUDA;
  // the block-word maps are not read with pre-arranged scales
  return launch_sd4_mx<false, false, true, true>(xa, xa, xa, xa, xa, wb, bias_bf16, M, N, K,
                                                 out_bf16, stream, K / G::BK, nullptr, 0,
                                                 x_tiles, w_tiles);
}

qs_status qs_sd4_decode(const void* codes, const uint16_t* meta, int64_t rows, int64_t K,
                        void* out_bf16, void* stream) {
  if (!codes || !meta || !out_bf16) return QS_ERR_NULL;
  if (rows <= 0 || K <= 0 || K % 256 != 0) return QS_ERR_SHAPE;
  if (K > QS_MAX_K || rows > QS_MAX_ROWS) return QS_ERR_RANGE;
  if (!aligned16(codes) || !aligned16(meta) || !aligned16(out_bf16)) return QS_ERR_ALIGN;
  for (const void* p : {codes, static_cast<const void*>(meta), static_cast<const void*>(out_bf16)})
    QS_TRY(check_device_ptr(p));
  const int sms = qs::sm_count();
  if (sms <= 0) return QS_ERR_CUDA;
  const int64_t tasks = rows * (K / 16);
  int64_t grid = (tasks + 255) / 256;
  if (grid > static_cast<int64_t>(sms) * 8) grid = static_cast<int64_t>(sms) * 8;
  qs::sd4::gemm_sd4::sd4_decode_kernel<<<static_cast<unsigned>(grid), 256, 0,
                                         static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(codes), meta, rows, static_cast<int>(K),
      static_cast<uint16_t*>(out_bf16));
  return cudaGetLastError() == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}

qs_status qs_sd4_linear_wdec(const void* x_codes, const uint16_t* x_meta, const void* w_bf16,
                             const void* bias_bf16, int64_t M, int64_t N, int64_t K,
                             void* out_bf16, void* stream) {
  namespace G = qs::sd4::gemm_sd4;
  if (!x_codes || !x_meta || !w_bf16 || !out_bf16) return QS_ERR_NULL;
  if (M <= 0 || N <= 0 || K <= 0 || K % 256 != 0 || N % 16 != 0) return QS_ERR_SHAPE;
  if (K > QS_MAX_K || M > INT32_MAX || N > INT32_MAX) return QS_ERR_RANGE;
  if (!aligned16(x_codes) || !aligned16(x_meta) || !aligned16(w_bf16) || !aligned16(out_bf16) ||
      (bias_bf16 && !aligned16(bias_bf16)))
    return QS_ERR_ALIGN;
  for (const void* p : {x_codes, static_cast<const void*>(x_meta), w_bf16,
                        static_cast<const void*>(out_bf16)})
    QS_TRY(check_device_ptr(p));
  if (bias_bf16) QS_TRY(check_device_ptr(bias_bf16));
  CUtensorMap ca, ma, wb;
  if (!qs::make_tensor_map_2d(&ca, x_codes, static_cast<uint64_t>(K) / 2,
                              static_cast<uint64_t>(M), G::BK / 2, G::BM, false) ||
      !qs::make_tensor_map_2d(&ma, x_meta, static_cast<uint64_t>(K) / 16,
                              static_cast<uint64_t>(M), 16, G::BM, false) ||
      !qs::make_tensor_map_2d(&wb, w_bf16, static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                              G::BK, G::BN, true, 2))
    return QS_ERR_CUDA;
  return launch_sd4_gemm<true>(ca, ca, ma, ma, wb, bias_bf16, M, N, K, out_bf16, stream);
}

qs_status qs_sd4_quant_decomp(const void* x_bf16, int64_t M, int64_t K, const int32_t* rows,
                              int64_t S, void* codes2, uint16_t* meta2, void* stream) {
  if (!x_bf16 || !rows || !codes2 || !meta2) return QS_ERR_NULL;
  if (M <= 0 || S <= 0 || K <= 0 || K % 256 != 0) return QS_ERR_SHAPE;
  if (2 * K > QS_MAX_K || M > INT32_MAX || S > QS_MAX_ROWS) return QS_ERR_RANGE;
  if (!aligned16(x_bf16) || !aligned16(codes2) || !aligned16(meta2) ||
      (reinterpret_cast<uintptr_t>(rows) & 3u))
    return QS_ERR_ALIGN;
  for (const void* p : {x_bf16, static_cast<const void*>(rows), static_cast<const void*>(codes2),
                        static_cast<const void*>(meta2)})
    QS_TRY(check_device_ptr(p));
  const int sms = qs::sm_count();
  if (sms <= 0) return QS_ERR_CUDA;
  const int64_t chunks = S * (K / 256);
  int64_t grid = (chunks + qs::sd4::kWarps - 1) / qs::sd4::kWarps;
  if (grid > static_cast<int64_t>(sms) * 4) grid = static_cast<int64_t>(sms) * 4;
  qs::sd4::sd4_decomp_kernel<<<static_cast<unsigned>(grid), qs::sd4::kThreads, 0,
                               static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(x_bf16), M, static_cast<int>(K), rows, S,
      static_cast<uint8_t*>(codes2), meta2);
  return cudaGetLastError() == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}

qs_status qs_sd4_linear_decomp(const void* codes2, const uint16_t* meta2, const int32_t* rows,
                               int64_t S, const void* w_codes, const uint16_t* w_meta,
                               const void* w_e4m3, const void* bias_bf16, int64_t M, int64_t N,
                               int64_t K, void* out_bf16, void* stream) {
  if (!codes2 || !meta2 || !rows || !out_bf16 || !w_meta) return QS_ERR_NULL;
  if (!w_e4m3 && !w_codes) return QS_ERR_NULL;
  if (M <= 0 || S <= 0 || N <= 0 || K <= 0 || K % 256 != 0 || N % 16 != 0) return QS_ERR_SHAPE;
  if (2 * K > QS_MAX_K || M > INT32_MAX || S > INT32_MAX || N > INT32_MAX) return QS_ERR_RANGE;
  if (!aligned16(codes2) || !aligned16(meta2) || !aligned16(out_bf16) || !aligned16(w_meta) ||
      (reinterpret_cast<uintptr_t>(rows) & 3u) || (bias_bf16 && !aligned16(bias_bf16)))
    return QS_ERR_ALIGN;
  if (w_e4m3 ? !aligned16(w_e4m3) : !aligned16(w_codes)) return QS_ERR_ALIGN;
  for (const void* p : {codes2, static_cast<const void*>(meta2), static_cast<const void*>(rows),
                        static_cast<const void*>(out_bf16), static_cast<const void*>(w_meta),
                        w_e4m3 ? w_e4m3 : w_codes})
    QS_TRY(check_device_ptr(p));
  if (bias_bf16) QS_TRY(check_device_ptr(bias_bf16));
  // A: S rows of 2K codes; the weights' K walked twice
  return run_sd4_mx(codes2, nullptr, meta2, S, 2 * K, w_e4m3 ? nullptr : w_codes, w_e4m3, w_meta,
                    bias_bf16, N, K, out_bf16, stream, rows, M);
}

qs_status qs_gelu_bf16(const void* x_bf16, int64_t n, void* y_bf16, void* stream) {
  if (!x_bf16 || !y_bf16) return QS_ERR_NULL;
  if (n <= 0) return QS_ERR_SHAPE;
  if (!aligned16(x_bf16) || !aligned16(y_bf16)) return QS_ERR_ALIGN;
  QS_TRY(check_device_ptr(x_bf16));
  QS_TRY(check_device_ptr(y_bf16));
  const int sms = qs::sm_count();
  if (sms <= 0) return QS_ERR_CUDA;
  const int64_t nvec = n / 8;
  if (n >= qs::kGeluTableMinElems) {
    // one CTA per SM (the 128 KB table), each building its own table
    if (cudaFuncSetAttribute(qs::gelu_bf16_table_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             qs::kGeluTableBytes) != cudaSuccess)
      return QS_ERR_CUDA;
    qs::gelu_bf16_table_kernel<<<static_cast<unsigned>(sms), qs::kGeluTableThreads,
                                 qs::kGeluTableBytes, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint16_t*>(x_bf16), n, static_cast<uint16_t*>(y_bf16));
    return cudaGetLastError() == cudaSuccess ? QS_OK : QS_ERR_CUDA;
  }
  int64_t blocks = (nvec + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  qs::gelu_bf16_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(x_bf16), n, static_cast<uint16_t*>(y_bf16));
  return cudaGetLastError() == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}

qs_status qs_linear_noalloc(const void* x_bf16, int64_t M, int64_t K, float alpha,
                            const void* w_packed, const float* w_scale, const void* bias_bf16,
                            int64_t N, int bits, void* out_bf16, void* stream) {
  const int64_t need = qs_linear_workspace_bytes(M, K, bits);
  if (need < 0) return check_bits(bits) != QS_OK ? QS_ERR_BITS : QS_ERR_SHAPE;
  if (need > static_cast<int64_t>(QS_NOALLOC_SCRATCH_BYTES)) return QS_ERR_RANGE;
  void* scratch = noalloc_scratch_address();
  if (!scratch) return QS_ERR_CUDA;
  return qs_linear(x_bf16, M, K, alpha, w_packed, w_scale, bias_bf16, N, bits, scratch,
                   static_cast<int64_t>(QS_NOALLOC_SCRATCH_BYTES), out_bf16, stream);
}

qs_status qs_selftest_timeout(int64_t timeout_us, void* stream) {
  if (timeout_us < 1 || timeout_us > 1000000) return QS_ERR_RANGE;
  qs::selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(timeout_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}

qs_status qs_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return QS_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, qs::g_error_word, sizeof(word)) != cudaSuccess)
    return QS_ERR_CUDA;
  if (word) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(qs::g_error_word, &zero, sizeof(zero)) != cudaSuccess)
      return QS_ERR_CUDA;
    return (word & ~static_cast<unsigned int>(qs::kErrIndex)) ? QS_ERR_TIMEOUT : QS_ERR_RANGE;
  }
  return QS_OK;
}

const char* qs_status_str(int status) {
  switch (status) {
    case QS_OK: return "ok";
    case QS_ERR_NULL: return "a required pointer is NULL";
    case QS_ERR_SHAPE: return "bad shape (need M,N,K > 0, K % 128 == 0, N % 16 == 0)";
    case QS_ERR_BITS: return "bits must be 4, 6 or 8";
    case QS_ERR_ALIGN: return "pointer not 16-byte aligned";
    case QS_ERR_RANGE: return "value out of range (alpha, flags or a size limit)";
    case QS_ERR_CUDA: return "CUDA call or launch failed";
    case QS_ERR_TIMEOUT: return "a kernel wait exceeded its bound";
    case QS_ERR_PTR: return "pointer is not device memory of the current device";
    default: return "unknown status";
  }
}

const char* qs_version(void) { return "qs 0.2.0 sm_100a"; }

}  // extern "C"
