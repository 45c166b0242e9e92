// Elementwise GELU between the ffn-up and ffn-down linears of a transformer
// block chain (bf16 in, bf16 out; exact-erf form evaluated in binary32).
// GELU(x) = x * Phi(x) with Phi(x) = erfc(-x / sqrt(2)) / 2: written with erfc
// so that the tail x << 0 keeps its relative accuracy (1 + erf(x/sqrt(2))
// cancels to 0 there).
#pragma once

#include <cuda_bf16.h>

#include "qs_ptx.cuh"

namespace qs {

// GELU of the bf16 number with bit pattern `xb` (low 16 bits), as a bf16
// bit pattern.  Both kernels below evaluate it through this one function.
__device__ __forceinline__ uint32_t gelu_bf16_bits(uint32_t xb) {
  const float a = __uint_as_float(xb << 16);
  const float g = 0.5f * a * erfcf(-a * 0.70710678118654752f);
  const __nv_bfloat16 r = __float2bfloat16_rn(g);
  return static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&r));
}

// Direct evaluation, 8 elements per thread per step (short inputs).
__global__ void __launch_bounds__(256) gelu_bf16_kernel(const uint16_t* x, int64_t n,
                                                        uint16_t* y) {
  const int64_t nvec = n / 8;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nvec;
       i += stride) {
    const uint4 d = *reinterpret_cast<const uint4*>(x + i * 8);
    const uint32_t in[4] = {d.x, d.y, d.z, d.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      o[k] = gelu_bf16_bits(in[k] & 0xFFFFu) | (gelu_bf16_bits(in[k] >> 16) << 16);
    *reinterpret_cast<uint4*>(y + i * 8) = make_uint4(o[0], o[1], o[2], o[3]);
  }
  // tail (n % 8 elements), handled by the first threads of block 0
  const int64_t t = nvec * 8 + threadIdx.x;
  if (blockIdx.x == 0 && t < n) y[t] = static_cast<uint16_t>(gelu_bf16_bits(x[t]));
}

// Long inputs: a bf16 input takes one of 65536 bit patterns, so each CTA
// first evaluates gelu_bf16_bits for every pattern into a 128 KB shared-memory
// table (64 evaluations per thread) and then streams the tensor with one table
// read per element.  The results are those of the direct kernel by
// construction; the stream is bound by HBM instead of by the erfc arithmetic.
constexpr int kGeluTableThreads = 1024;
constexpr int kGeluTableBytes = 65536 * 2;
constexpr int64_t kGeluTableMinElems = int64_t{1} << 24;  // below: direct kernel

__device__ __forceinline__ uint32_t gelu_lookup2(const uint16_t* tab, uint32_t w) {
  return static_cast<uint32_t>(tab[w & 0xFFFFu]) | (static_cast<uint32_t>(tab[w >> 16]) << 16);
}

__device__ __forceinline__ uint4 gelu_lookup8(const uint16_t* tab, uint4 d) {
  return make_uint4(gelu_lookup2(tab, d.x), gelu_lookup2(tab, d.y), gelu_lookup2(tab, d.z),
                    gelu_lookup2(tab, d.w));
}

__global__ void __launch_bounds__(kGeluTableThreads, 1)
    gelu_bf16_table_kernel(const uint16_t* x, int64_t n, uint16_t* y) {  // x and y may alias
  extern __shared__ __align__(16) uint16_t gelu_tab[];
  for (int i = threadIdx.x; i < 65536; i += blockDim.x)
    gelu_tab[i] = static_cast<uint16_t>(gelu_bf16_bits(static_cast<uint32_t>(i)));
  __syncthreads();
  const uint16_t* tab = gelu_tab;
  const int64_t nvec = n / 8;
  const uint4* xv = reinterpret_cast<const uint4*>(x);
  uint4* yv = reinterpret_cast<uint4*>(y);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  // four independent 16-byte loads in flight per thread
  for (; i + 3 * stride < nvec; i += 4 * stride) {
    uint4 d[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) d[u] = __ldcs(xv + i + u * stride);
#pragma unroll
    for (int u = 0; u < 4; ++u) __stcs(yv + i + u * stride, gelu_lookup8(tab, d[u]));
  }
  for (; i < nvec; i += stride) __stcs(yv + i, gelu_lookup8(tab, __ldcs(xv + i)));
  const int64_t t = nvec * 8 + threadIdx.x;
  if (blockIdx.x == 0 && t < n) y[t] = tab[x[t]];
}

// Diagnostic: waits on an mbarrier that nothing ever arrives on, with a
// bounded wait; the wait gives up after `limit_ns` and records the timeout in
// the library's device error word.  Exercises the failure path of the bounded
// waits without faulting or hanging the GPU.
__global__ void selftest_timeout_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_mbar_init();
    mbar_wait_limit(b, 0, limit_ns, kErrSelfTest);
  }
}

}  // namespace qs
