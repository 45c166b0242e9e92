// δ-guided bit switching on the device (DVD-Quant, "Resumen técnico" §2.C):
// the normalised L1 change between consecutive outputs of a layer is
// accumulated, and the width of the layer's next step (4 or 8 bits) is chosen
// from the accumulator without a round trip to the host.
//
//   d = sum |y_cur - y_prev| / sum |y_prev|     (binary64 terms and sums)
//   acc += d;  next = acc < delta ? 4 : 8;  acc = 0 when switching to 8
//
// The first step has no previous output: it only records that a step ran,
// and the next width follows from the unchanged accumulator.
//
// The reduction reads both outputs once (16-byte loads, grid-stride, two
// strides per iteration), each thread sums its elements in a fixed order, blocks reduce through shared
// memory in a fixed tree and write one partial pair each; the last block to
// finish (a counter in the state) adds the partials in block order.  With the
// grid fixed by the device's SM count the result is the same on every run.
#pragma once

#include <cstdint>

#include "qs.h"

namespace qs {
namespace gbs {

constexpr int kThreads = 256;
constexpr int kMaxBlocks = QS_GBS_MAX_BLOCKS;

__device__ __forceinline__ double bf16_to_f64(uint32_t h) {
  return static_cast<double>(__uint_as_float(h << 16));
}

// Adds |a - b| and |b| of the 8 bf16 pairs in (a, b) to the running sums.
__device__ __forceinline__ void accumulate8(const uint4 a, const uint4 b, double& num,
                                            double& den) {
  const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
  const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const double a0 = bf16_to_f64(aw[k] & 0xFFFFu), a1 = bf16_to_f64(aw[k] >> 16);
    const double b0 = bf16_to_f64(bw[k] & 0xFFFFu), b1 = bf16_to_f64(bw[k] >> 16);
    num += fabs(a0 - b0);
    den += fabs(b0);
    num += fabs(a1 - b1);
    den += fabs(b1);
  }
}

// Block-wide sum of (num, den) in a fixed tree: warp shuffles, then warp 0.
__device__ __forceinline__ void block_sum(double& num, double& den) {
  __shared__ double s_num[kThreads / 32], s_den[kThreads / 32];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    num += __shfl_xor_sync(0xffffffffu, num, off);
    den += __shfl_xor_sync(0xffffffffu, den, off);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    s_num[warp] = num;
    s_den[warp] = den;
  }
  __syncthreads();
  if (warp == 0) {
    num = lane < kThreads / 32 ? s_num[lane] : 0.0;
    den = lane < kThreads / 32 ? s_den[lane] : 0.0;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      num += __shfl_xor_sync(0xffffffffu, num, off);
      den += __shfl_xor_sync(0xffffffffu, den, off);
    }
  }
}

// The decision after one step (the distance d, or no distance at the first step).
__device__ __forceinline__ void decide(qs_gbs_state* st, double d, bool have_d, double delta) {
  double acc = st->acc;
  if (have_d) acc += d;
  st->last_d = have_d ? d : -1.0;
  if (acc < delta) {
    st->acc = acc;
    st->bits = 4;
  } else {
    st->acc = 0.0;
    st->bits = 8;
  }
  st->step += 1;
}

__global__ void __launch_bounds__(kThreads) gbs_update_kernel(const uint16_t* __restrict__ cur,
                                                              const uint16_t* __restrict__ prev,
                                                              int64_t n, double delta,
                                                              qs_gbs_state* st) {
  double num = 0.0, den = 0.0;
  const int64_t nvec = n / 8;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  const uint4* a4 = reinterpret_cast<const uint4*>(cur);
  const uint4* b4 = reinterpret_cast<const uint4*>(prev);
  // two grid strides per iteration: four 16-byte loads in flight per thread
  // (0.94 of the measured HBM bandwidth against 0.81 with one stride; four
  // strides measured slower)
  int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  for (; i + stride < nvec; i += 2 * stride) {
    const uint4 a0 = __ldcs(a4 + i), b0 = __ldcs(b4 + i);
    const uint4 a1 = __ldcs(a4 + i + stride), b1 = __ldcs(b4 + i + stride);
    accumulate8(a0, b0, num, den);
    accumulate8(a1, b1, num, den);
  }
  if (i < nvec) accumulate8(__ldcs(a4 + i), __ldcs(b4 + i), num, den);
  // the last n % 8 elements: thread 0 of block 0
  if (blockIdx.x == 0 && threadIdx.x == 0)
    for (int64_t i = nvec * 8; i < n; ++i) {
      const double a = bf16_to_f64(cur[i]), b = bf16_to_f64(prev[i]);
      num += fabs(a - b);
      den += fabs(b);
    }
  block_sum(num, den);
  __shared__ bool s_last;
  if (threadIdx.x == 0) {
    st->partial[0][blockIdx.x] = num;
    st->partial[1][blockIdx.x] = den;
    __threadfence();
    s_last = atomicAdd(&st->blocks_done, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last || threadIdx.x != 0) return;
  __threadfence();
  const volatile double* pn = st->partial[0];
  const volatile double* pd = st->partial[1];
  double tn = 0.0, td = 0.0;
  for (unsigned b = 0; b < gridDim.x; ++b) {
    tn += pn[b];
    td += pd[b];
  }
  double d;
  if (td == 0.0)
    d = tn == 0.0 ? 0.0 : __longlong_as_double(0x7FF0000000000000ll);  // +inf
  else
    d = tn / td;
  st->blocks_done = 0u;
  decide(st, d, true, delta);
}

// The first step: no previous output, no distance.
__global__ void gbs_first_kernel(double delta, qs_gbs_state* st) { decide(st, 0.0, false, delta); }

__global__ void gbs_reset_kernel(qs_gbs_state* st) {
  st->acc = 0.0;
  st->last_d = -1.0;
  st->bits = 8;
  st->step = 0;
  st->blocks_done = 0u;
}

}  // namespace gbs
}  // namespace qs
