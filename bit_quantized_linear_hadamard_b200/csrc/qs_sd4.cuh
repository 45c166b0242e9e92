// SD4: SemanticDialect's mixed-format 4-bit block quantisation ("Resumen
// técnico" §2.A): 32 candidate 4-bit formats ("dialects"), one chosen per
// block of 32 elements through precomputed tables, a power-of-two scale per
// block that normalises the magnitudes to [0, 2).
//
// This implementation's formatbook (the pages print none): a code is a sign
// bit and a 3-bit level index; dialect d = 8a + s has the magnitudes L/8 with
// top level t = 15 - a and, for i = 1..7,
//   L = floor((2 t (49 p i + 7 q i^2 + r i^3) + 2744) / 5488)
// raised to be strictly increasing, for the shape (p, q, r) = kShapes[s]; L0 = 0.
// Block: e = max(floor(log2 amax), -126) (0 for a zero block); bin of an
// element b = min(floor(|x| 2^(7-e)), 255); Qerror[d][b] = min_i
// (2b + 1 - 32 L_i)^2, Qvalue[d][b] = that i; the block's dialect is
// argmin_d sum Qerror[d][b_k] (the smallest d on ties); code =
// (x < 0) << 3 | Qvalue[d][b].  Stored: codes two per byte (element 2j in the
// low nibble), one 16-bit word per block (low byte e as int8, high byte d).
//
// Quantiser: persistent CTAs of 8 warps; each CTA first builds the tables in
// shared memory.  A warp takes 8 blocks (256 elements) at a time: each lane
// loads 8 elements (16 bytes), four lanes reduce a block's absmax, and the
// bins go to shared memory; then for each block lane d sums dialect d's cost
// (conflict-free: the table is laid out [bin][dialect]) and a warp minimum on
// (cost << 5 | d) picks the dialect; finally each lane writes its 8 codes.
#pragma once

#include <cstdint>

namespace qs {
namespace sd4 {

constexpr int kBlock = 32;
constexpr int kDialects = 32;
constexpr int kBins = 256;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__host__ __device__ constexpr int shape_coef(int s, int k) {
  // (p, q, r) per shape: ramp, square, cube weights (sum 8)
  constexpr int kShapes[8][3] = {{8, 0, 0}, {6, 2, 0}, {4, 4, 0}, {3, 5, 0},
                                 {2, 5, 1}, {0, 8, 0}, {1, 3, 4}, {0, 3, 5}};
  return kShapes[s][k];
}

// Level L[d][i] of the formatbook (i = 0..7).
__host__ __device__ inline int level(int d, int i) {
  const int t = 15 - d / 8, s = d % 8;
  int prev = 0;
  for (int j = 1; j <= i; ++j) {
    const int p = shape_coef(s, 0), q = shape_coef(s, 1), r = shape_coef(s, 2);
    int v = (2 * t * (49 * p * j + 7 * q * j * j + r * j * j * j) + 2744) / 5488;
    if (v < prev + 1) v = prev + 1;
    prev = v;
  }
  return i == 0 ? 0 : prev;
}

struct Tables {
  uint32_t qerr[kBins][kDialects];  // [bin][dialect]: lane d reads word d
  uint8_t qval[kDialects][kBins];
};

__device__ void build_tables(Tables* tb) {
  for (int idx = threadIdx.x; idx < kDialects * kBins; idx += blockDim.x) {
    const int d = idx / kBins, b = idx % kBins;
    uint32_t best = 0xFFFFFFFFu;
    int bi = 0;
    for (int i = 0; i < 8; ++i) {
      const int diff = 2 * b + 1 - 32 * level(d, i);
      const uint32_t sq = static_cast<uint32_t>(diff * diff);
      if (sq < best) {
        best = sq;
        bi = i;
      }
    }
    tb->qerr[b][d] = best;
    tb->qval[d][b] = static_cast<uint8_t>(bi);
  }
}

// 2^n as binary32 for n in [-127, 127] (n = -127: the subnormal 2^-127).
__device__ __forceinline__ float pow2f(int n) {
  return n >= -126 ? __int_as_float((n + 127) << 23) : __int_as_float(0x00400000);
}

__global__ void __launch_bounds__(kThreads) sd4_quant_kernel(const uint16_t* __restrict__ x,
                                                            int64_t rows, int K,
                                                            uint8_t* __restrict__ codes,
                                                            uint16_t* __restrict__ meta) {
  __shared__ Tables tb;
  __shared__ uint8_t s_bins[kWarps][8][kBlock];
  build_tables(&tb);
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blocks_per_row = K / kBlock;
  const int64_t chunks_per_row = K / 256;  // 8 blocks per chunk (K % 256 == 0)
  const int64_t num_chunks = rows * chunks_per_row;
  for (int64_t c = static_cast<int64_t>(blockIdx.x) * kWarps + warp; c < num_chunks;
       c += static_cast<int64_t>(gridDim.x) * kWarps) {
    const int64_t row = c / chunks_per_row;
    const int col0 = static_cast<int>(c % chunks_per_row) * 256;
    const int blk = lane >> 2;  // block within the chunk
    // 8 elements of block blk: elements 8 * (lane & 3) .. + 7
    const uint4 raw =
        __ldg(reinterpret_cast<const uint4*>(x + row * static_cast<int64_t>(K) + col0) + lane);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    float a[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      a[2 * k] = __uint_as_float(w[k] << 16);
      a[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fabsf(a[k]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    int e = 0;
    if (amax != 0.f) {
      const int ef = (__float_as_uint(amax) >> 23) & 0xFF;
      e = ef == 0 ? -126 : max(ef - 127, -126);
    }
    const float sc = pow2f(-e);  // exact; |x| 2^-e < 2
    uint8_t bins[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float v = __fmul_rn(__fmul_rn(fabsf(a[k]), sc), 128.f);
      const int b = static_cast<int>(v);  // truncation = floor for v >= 0
      bins[k] = static_cast<uint8_t>(b > 255 ? 255 : b);
    }
    *reinterpret_cast<uint2*>(&s_bins[warp][blk][8 * (lane & 3)]) =
        make_uint2(bins[0] | (bins[1] << 8) | (bins[2] << 16) | (static_cast<uint32_t>(bins[3]) << 24),
                   bins[4] | (bins[5] << 8) | (bins[6] << 16) | (static_cast<uint32_t>(bins[7]) << 24));
    __syncwarp();
    // dialect choice: lane = dialect
    int my_d = 0;
#pragma unroll 1
    for (int j = 0; j < 8; ++j) {
      uint32_t cost = 0;
#pragma unroll 8
      for (int k = 0; k < kBlock; ++k) cost += tb.qerr[s_bins[warp][j][k]][lane];
      uint32_t key = (cost << 5) | static_cast<uint32_t>(lane);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) key = min(key, __shfl_xor_sync(0xffffffffu, key, off));
      if (j == blk) my_d = static_cast<int>(key & 31u);
    }
    // codes of this lane's 8 elements
    uint32_t packed = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t code = (a[k] < 0.f ? 8u : 0u) | tb.qval[my_d][bins[k]];
      packed |= code << (4 * k);
    }
    const int64_t code_off = row * static_cast<int64_t>(K / 2) + col0 / 2 + 4 * lane;
    *reinterpret_cast<uint32_t*>(codes + code_off) = packed;
    if ((lane & 3) == 0)
      meta[row * blocks_per_row + col0 / kBlock + blk] =
          static_cast<uint16_t>((static_cast<uint32_t>(e) & 0xFFu) | (static_cast<uint32_t>(my_d) << 8));
    __syncwarp();  // s_bins is rewritten by the next chunk
  }
}

}  // namespace sd4
}  // namespace qs
