// Bounded-init grid refinement of the weights (DVD-Quant, "Resumen técnico"
// §2.A): offline, per output channel, an asymmetric b-bit grid
// (step Δ, integer zero point z) for the rotated weight row u:
//   1. bound search: for j = 0..J-1 the bounds r_j·[min u, max u] with
//      r_j = 1 - j/(2J) give Δ = (hi - lo)/(2^b - 1), z = clamp(rint(-lo/Δ));
//      the grid with the smallest squared error wins (first on ties);
//   2. T refits: the closed-form least-squares fit u ≈ Δ q + c to the current
//      codes, z = clamp(rint(-c/Δ)), Δ refit for that z, re-quantise; the
//      grid with the smallest error over all steps is kept.
// Codes q = clamp(rint(fl(u · fl(1/Δ))) + z, 0, 2^b - 1); error
// sum (u - fl(Δ (q - z)))^2.  Every sum runs in index order in binary64 and
// every product, sum and quotient is a separately rounded binary64 operation
// (the __d*_rn intrinsics keep the compiler from fusing them), so every
// integer decision is reproducible.  Stored: signed codes q - 2^(b-1)
// (nibbles or bytes), scale fl32(Δ)·scale_mul and offset 2^(b-1) - z.
//
// One CTA per row; the row lives in shared memory (binary32, 4 bytes per
// element), the block Walsh-Hadamard transform runs there with one thread per
// 128-block in the butterfly order h = 1, 2, ..., 64, the candidates run one
// per thread, the refits in one thread.  Offline work: simple over fast.
#pragma once

#include <cstdint>

namespace qs {
namespace bgr {

constexpr int kThreads = 256;
constexpr int kMaxCandidates = kThreads;
constexpr int kMaxK = 32768;  // the row in shared memory: 4 bytes per element

struct Grid {
  double step;
  int zero;
};

__device__ __forceinline__ int grid_code(float u, double inv, int zero, int levels) {
  const double r = rint(__dmul_rn(static_cast<double>(u), inv));
  const double q = fmin(fmax(__dadd_rn(r, static_cast<double>(zero)), 0.0),
                        static_cast<double>(levels));
  return static_cast<int>(q);
}

// Squared error of a grid over the row, index order.
__device__ double grid_error(const float* u, int K, Grid g, int levels) {
  const double inv = __ddiv_rn(1.0, g.step);
  double acc = 0.0;
  for (int k = 0; k < K; ++k) {
    const int q = grid_code(u[k], inv, g.zero, levels);
    const double dq = __dmul_rn(g.step, static_cast<double>(q - g.zero));
    const double e = __dsub_rn(static_cast<double>(u[k]), dq);
    acc = __dadd_rn(acc, __dmul_rn(e, e));
  }
  return acc;
}

__device__ Grid grid_from_bounds(double lo, double hi, int levels) {
  Grid g;
  g.step = __ddiv_rn(__dsub_rn(hi, lo), static_cast<double>(levels));
  const double z = rint(__ddiv_rn(-lo, g.step));
  g.zero = static_cast<int>(fmin(fmax(z, 0.0), static_cast<double>(levels)));
  return g;
}

// Least-squares refit from the codes of grid `cur` (recomputed here); false
// when the fit is degenerate.
__device__ bool least_squares(const float* u, int K, Grid cur, int levels, double su, Grid* out) {
  const double inv = __ddiv_rn(1.0, cur.step);
  long long sq = 0, sqq = 0;
  double squ = 0.0;
  for (int k = 0; k < K; ++k) {
    const int q = grid_code(u[k], inv, cur.zero, levels);
    sq += q;
    sqq += static_cast<long long>(q) * q;
    squ = __dadd_rn(squ, __dmul_rn(static_cast<double>(q), static_cast<double>(u[k])));
  }
  const double n = static_cast<double>(K);
  const double dsq = static_cast<double>(sq), dsqq = static_cast<double>(sqq);
  const double den = __dsub_rn(__dmul_rn(n, dsqq), __dmul_rn(dsq, dsq));
  if (den == 0.0) return false;
  double step = __ddiv_rn(__dsub_rn(__dmul_rn(n, squ), __dmul_rn(dsq, su)), den);
  if (!(step > 0.0)) return false;
  const double c = __ddiv_rn(__dsub_rn(su, __dmul_rn(step, dsq)), n);
  const double zr = rint(__ddiv_rn(-c, step));
  const int z = static_cast<int>(fmin(fmax(zr, 0.0), static_cast<double>(levels)));
  // refit the step for the integer zero point, the same codes
  long long tt = 0;
  double sut = 0.0;
  for (int k = 0; k < K; ++k) {
    const int t = grid_code(u[k], inv, cur.zero, levels) - z;
    tt += static_cast<long long>(t) * t;
    sut = __dadd_rn(sut, __dmul_rn(static_cast<double>(u[k]), static_cast<double>(t)));
  }
  if (tt == 0) return false;
  step = __ddiv_rn(sut, static_cast<double>(tt));
  if (!(step > 0.0)) return false;
  out->step = step;
  out->zero = z;
  return true;
}

template <int BITS>
__global__ void __launch_bounds__(kThreads) bgr_pack_kernel(
    const uint16_t* __restrict__ w, int K, int rotate, int candidates, int iterations,
    float scale_mul, uint8_t* __restrict__ packed, float* __restrict__ scale_out,
    int* __restrict__ offset_out) {
  constexpr int kLevels = (1 << BITS) - 1;
  constexpr int kHalf = 1 << (BITS - 1);
  extern __shared__ __align__(16) float u[];
  __shared__ double s_err[kMaxCandidates];
  __shared__ Grid s_grid[kMaxCandidates];
  __shared__ float s_lo[kThreads / 32], s_hi[kThreads / 32];
  __shared__ Grid s_best;

  const int64_t row = blockIdx.x;
  const uint16_t* wr = w + row * static_cast<int64_t>(K);
  for (int k = threadIdx.x; k < K; k += kThreads)
    u[k] = __uint_as_float(static_cast<uint32_t>(wr[k]) << 16);
  __syncthreads();

  if (rotate) {  // one 128-block per thread, butterfly stages h = 1..64
    for (int b = threadIdx.x; b < K / 128; b += kThreads) {
      float* v = u + b * 128;
      for (int h = 1; h < 128; h <<= 1)
        for (int i = 0; i < 128; ++i)
          if ((i & h) == 0) {
            const float a = v[i], c = v[i + h];
            v[i] = __fadd_rn(a, c);
            v[i + h] = __fsub_rn(a, c);
          }
    }
    __syncthreads();
  }

  // min and max of the row (order-independent)
  float lo = u[0], hi = u[0];
  for (int k = threadIdx.x; k < K; k += kThreads) {
    lo = fminf(lo, u[k]);
    hi = fmaxf(hi, u[k]);
  }
  for (int off = 16; off > 0; off >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
  }
  if ((threadIdx.x & 31) == 0) {
    s_lo[threadIdx.x >> 5] = lo;
    s_hi[threadIdx.x >> 5] = hi;
  }
  __syncthreads();
  lo = s_lo[0];
  hi = s_hi[0];
  for (int i = 1; i < kThreads / 32; ++i) {
    lo = fminf(lo, s_lo[i]);
    hi = fmaxf(hi, s_hi[i]);
  }

  if (hi == lo) {  // one level: Δ = |u0| (1 for a zero row), u0 itself a level
    if (threadIdx.x == 0) {
      Grid g;
      if (lo == 0.f) {
        g.step = 1.0;
        g.zero = 0;
      } else {
        g.step = fabs(static_cast<double>(lo));
        g.zero = lo > 0.f ? 0 : kLevels;
      }
      s_best = g;
    }
  } else {
    // bound search: one candidate per thread
    const int j = threadIdx.x;
    if (j < candidates) {
      const double r = __dsub_rn(1.0, __ddiv_rn(static_cast<double>(j),
                                                __dmul_rn(2.0, static_cast<double>(candidates))));
      const Grid g = grid_from_bounds(__dmul_rn(r, static_cast<double>(lo)),
                                      __dmul_rn(r, static_cast<double>(hi)), kLevels);
      s_grid[j] = g;
      s_err[j] = grid_error(u, K, g, kLevels);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int best = 0;
      for (int c = 1; c < candidates; ++c)
        if (s_err[c] < s_err[best]) best = c;
      Grid bg = s_grid[best];
      double be = s_err[best];
      // refits, index-order sums
      double su = 0.0;
      for (int k = 0; k < K; ++k) su = __dadd_rn(su, static_cast<double>(u[k]));
      Grid cur = bg;
      for (int it = 0; it < iterations; ++it) {
        Grid nxt;
        if (!least_squares(u, K, cur, kLevels, su, &nxt)) break;
        cur = nxt;
        const double e = grid_error(u, K, cur, kLevels);
        if (e < be) {
          be = e;
          bg = cur;
        }
      }
      s_best = bg;
    }
  }
  __syncthreads();

  // signed codes of the kept grid, packed like the symmetric path
  const Grid g = s_best;
  const double inv = __ddiv_rn(1.0, g.step);
  uint8_t* out = packed + row * static_cast<int64_t>(BITS == 4 ? K / 2 : K);
  if (BITS == 4) {
    for (int p = threadIdx.x; p < K / 2; p += kThreads) {
      const int s0 = grid_code(u[2 * p], inv, g.zero, kLevels) - kHalf;
      const int s1 = grid_code(u[2 * p + 1], inv, g.zero, kLevels) - kHalf;
      out[p] = static_cast<uint8_t>((s0 & 0xF) | ((s1 & 0xF) << 4));
    }
  } else {
    for (int k = threadIdx.x; k < K; k += kThreads)
      out[k] = static_cast<uint8_t>(grid_code(u[k], inv, g.zero, kLevels) - kHalf);
  }
  if (threadIdx.x == 0) {
    scale_out[row] = __fmul_rn(__double2float_rn(g.step), scale_mul);
    offset_out[row] = kHalf - g.zero;
  }
}

}  // namespace bgr
}  // namespace qs
