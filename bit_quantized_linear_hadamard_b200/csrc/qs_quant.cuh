// Fused rotate -> online scale -> quantize -> pack kernel (one row per CTA).
//
// DVD-Quant, "Resumen técnico" §2.B (ARQ): a Hadamard rotation spreads the
// extreme values across channels, and the quantization scale is computed at
// run time from the rotated values.  Serves both the per-token activation
// quantization (alpha = clip ratio) and the offline per-output-channel weight
// quantization (alpha = 1, scale multiplied by the exact 2^-7 that carries the
// two 1/sqrt(128) normalisations).
//
// Layout of the work: a row of K bf16 values is split in groups of 8
// consecutive elements (one 16-byte load each).  Thread t of a CTA of T
// threads owns groups t, t+T, ..., t+(G-1)T, so a warp reads 512 contiguous
// bytes per load instruction, and the 16 groups of one 128-element Hadamard
// block always sit in 16 consecutive lanes (T is a multiple of 32).  The
// butterfly stages h = 1, 2, 4 are done in registers, h = 8, 16, 32, 64 by
// xor-shuffles with lane distance 1, 2, 4, 8 — always in that order, so the
// binary32 roundings are those of the sequential butterfly.
#pragma once

#include "qs_ptx.cuh"

namespace qs {

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void butterfly(float& a, float& b) {
  const float t = a;
  a = __fadd_rn(t, b);
  b = __fsub_rn(t, b);
}

__device__ __forceinline__ void bf16x2_to_f32(uint32_t w, float& lo, float& hi) {
  lo = __uint_as_float(w << 16);
  hi = __uint_as_float(w & 0xFFFF0000u);
}

template <int G, int BITS, int MAXT>
__global__ void __launch_bounds__(MAXT) rotate_quant_kernel(const uint16_t* __restrict__ x, int K,
                                                            float alpha, float scale_mul,
                                                            int rotate, uint8_t* __restrict__ out,
                                                            float* __restrict__ scale_out) {
  constexpr int kQmax = BITS == 4 ? 7 : 127;
  __shared__ float warp_max[32];

  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int T = blockDim.x;
  const int ngroups = K >> 3;
  const uint16_t* xr = x + row * static_cast<int64_t>(K);

  float v[G][8];
#pragma unroll
  for (int j = 0; j < G; ++j) {
    const int g = tid + j * T;
    uint4 d = make_uint4(0u, 0u, 0u, 0u);
    if (g < ngroups) d = ld_stream_v4(xr + static_cast<int64_t>(g) * 8);
    bf16x2_to_f32(d.x, v[j][0], v[j][1]);
    bf16x2_to_f32(d.y, v[j][2], v[j][3]);
    bf16x2_to_f32(d.z, v[j][4], v[j][5]);
    bf16x2_to_f32(d.w, v[j][6], v[j][7]);
  }

  if (rotate) {
#pragma unroll
    for (int j = 0; j < G; ++j) {
      // h = 1
      butterfly(v[j][0], v[j][1]);
      butterfly(v[j][2], v[j][3]);
      butterfly(v[j][4], v[j][5]);
      butterfly(v[j][6], v[j][7]);
      // h = 2
      butterfly(v[j][0], v[j][2]);
      butterfly(v[j][1], v[j][3]);
      butterfly(v[j][4], v[j][6]);
      butterfly(v[j][5], v[j][7]);
      // h = 4
      butterfly(v[j][0], v[j][4]);
      butterfly(v[j][1], v[j][5]);
      butterfly(v[j][2], v[j][6]);
      butterfly(v[j][3], v[j][7]);
      // h = 8, 16, 32, 64: partner group is lane ^ 1, 2, 4, 8
#pragma unroll
      for (int m = 1; m <= 8; m <<= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float p = __shfl_xor_sync(0xffffffffu, v[j][e], m);
          v[j][e] = upper ? __fsub_rn(p, v[j][e]) : __fadd_rn(v[j][e], p);
        }
      }
    }
  }

  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < G; ++j)
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[j][e]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if (lane == 0) warp_max[tid >> 5] = amax;
  __syncthreads();
  amax = warp_max[0];
  for (int w = 1; w < (T >> 5); ++w) amax = fmaxf(amax, warp_max[w]);

  const float s = __fdiv_rn(__fmul_rn(alpha, amax), static_cast<float>(kQmax));
  if (tid == 0) scale_out[row] = __fmul_rn(s, scale_mul);
  const bool zero_scale = !(s > 0.f);

#pragma unroll
  for (int j = 0; j < G; ++j) {
    const int g = tid + j * T;
    if (g >= ngroups) continue;
    int q[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      int qi = 0;
      if (!zero_scale) {
        qi = __float2int_rn(__fdiv_rn(v[j][e], s));
        qi = min(max(qi, -kQmax), kQmax);
      }
      q[e] = qi;
    }
    if (BITS == 4) {
      uint32_t wv = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) wv |= (static_cast<uint32_t>(q[e]) & 0xFu) << (4 * e);
      *reinterpret_cast<uint32_t*>(out + row * static_cast<int64_t>(K >> 1) + g * 4) = wv;
    } else {
      uint2 wv;
      wv.x = (static_cast<uint32_t>(q[0]) & 0xFFu) | ((static_cast<uint32_t>(q[1]) & 0xFFu) << 8) |
             ((static_cast<uint32_t>(q[2]) & 0xFFu) << 16) | (static_cast<uint32_t>(q[3]) << 24);
      wv.y = (static_cast<uint32_t>(q[4]) & 0xFFu) | ((static_cast<uint32_t>(q[5]) & 0xFFu) << 8) |
             ((static_cast<uint32_t>(q[6]) & 0xFFu) << 16) | (static_cast<uint32_t>(q[7]) << 24);
      *reinterpret_cast<uint2*>(out + row * static_cast<int64_t>(K) + g * 8) = wv;
    }
  }
}

// Chooses (G groups per thread, T threads) for a row of `ngroups` 8-element
// groups: G <= 8, T a multiple of 32 and at most `max_t`, least idle slots,
// then the largest G.  Returns false if the row does not fit one pass.
inline bool choose_quant_shape(int ngroups, int max_t, int* G_out, int* T_out) {
  int best_g = 0, best_t = 0, best_waste = 1 << 30;
  for (int G = 8; G >= 1; --G) {
    int T = (ngroups + G - 1) / G;
    T = (T + 31) / 32 * 32;
    if (T > max_t) continue;
    const int waste = T * G - ngroups;
    if (waste < best_waste) {
      best_waste = waste;
      best_g = G;
      best_t = T;
    }
  }
  if (!best_g) return false;
  *G_out = best_g;
  *T_out = best_t;
  return true;
}

template <int BITS>
inline cudaError_t launch_rotate_quant_bits(const uint16_t* x, int64_t rows, int K, float alpha,
                                            float scale_mul, int rotate, uint8_t* out,
                                            float* scale, cudaStream_t stream) {
  // Rows up to 2048 groups (K <= 16384) run with at most 256 threads so each
  // thread may keep its 8*G values in registers; longer rows use up to 1024.
  const int ngroups = K / 8;
  const bool wide = ngroups > 256 * 8;
  int G = 0, T = 0;
  if (!choose_quant_shape(ngroups, wide ? 1024 : 256, &G, &T)) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(rows)), block(T);
#define QS_QUANT_CASE(GG)                                                                    \
  case GG:                                                                                   \
    if (wide)                                                                                \
      rotate_quant_kernel<GG, BITS, 1024>                                                    \
          <<<grid, block, 0, stream>>>(x, K, alpha, scale_mul, rotate, out, scale);          \
    else                                                                                     \
      rotate_quant_kernel<GG, BITS, 256>                                                     \
          <<<grid, block, 0, stream>>>(x, K, alpha, scale_mul, rotate, out, scale);          \
    break;
  switch (G) {
    QS_QUANT_CASE(1)
    QS_QUANT_CASE(2)
    QS_QUANT_CASE(3)
    QS_QUANT_CASE(4)
    QS_QUANT_CASE(5)
    QS_QUANT_CASE(6)
    QS_QUANT_CASE(7)
    QS_QUANT_CASE(8)
    default:
      return cudaErrorInvalidValue;
  }
#undef QS_QUANT_CASE
  return cudaGetLastError();
}

inline cudaError_t launch_rotate_quant(const uint16_t* x, int64_t rows, int K, int bits, float alpha,
                                       float scale_mul, int rotate, uint8_t* out, float* scale,
                                       cudaStream_t stream) {
  return bits == 4 ? launch_rotate_quant_bits<4>(x, rows, K, alpha, scale_mul, rotate, out, scale,
                                                 stream)
                   : launch_rotate_quant_bits<8>(x, rows, K, alpha, scale_mul, rotate, out, scale,
                                                 stream);
}

}  // namespace qs
