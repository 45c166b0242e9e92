// Elementwise GELU between the ffn-up and ffn-down linears of a transformer
// block chain (bf16 in, bf16 out; exact-erf form evaluated in binary32).
// GELU(x) = x * Phi(x) with Phi(x) = erfc(-x / sqrt(2)) / 2: written with erfc
// so that the tail x << 0 keeps its relative accuracy (1 + erf(x/sqrt(2))
// cancels to 0 there).
#pragma once

#include <cuda_bf16.h>

#include "qs_ptx.cuh"

namespace qs {

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
    for (int k = 0; k < 4; ++k) {
      const float a = __uint_as_float(in[k] << 16);
      const float b = __uint_as_float(in[k] & 0xFFFF0000u);
      const float ga = 0.5f * a * erfcf(-a * 0.70710678118654752f);
      const float gb = 0.5f * b * erfcf(-b * 0.70710678118654752f);
      const __nv_bfloat162 g = __floats2bfloat162_rn(ga, gb);
      o[k] = *reinterpret_cast<const uint32_t*>(&g);
    }
    *reinterpret_cast<uint4*>(y + i * 8) = make_uint4(o[0], o[1], o[2], o[3]);
  }
  // tail (n % 8 elements), handled by the first threads of block 0
  const int64_t t = nvec * 8 + threadIdx.x;
  if (blockIdx.x == 0 && t < n) {
    const float a = __uint_as_float(static_cast<uint32_t>(x[t]) << 16);
    const float ga = 0.5f * a * erfcf(-a * 0.70710678118654752f);
    const __nv_bfloat16 g = __float2bfloat16_rn(ga);
    y[t] = *reinterpret_cast<const uint16_t*>(&g);
  }
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
