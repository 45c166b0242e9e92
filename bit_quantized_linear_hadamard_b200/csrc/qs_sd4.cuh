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
// Quantiser (tc::sd4_quant_tc_kernel): one thread per block, the dialect
// choice as an exact integer product on the tensor cores (see there).  The
// activation decomposition uses a warp-level form (quant_warp_chunk): a warp
// takes 8 blocks (256 elements), four lanes reduce a block's absmax, and the
// half-warps score two blocks at a time on packed 16-bit Qerror pairs (see
// Tables), a warp minimum on (cost << 5 | d) picking the dialect.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "qs_ptx.cuh"

namespace qs {
namespace sd4 {

constexpr int kBlock = 32;
constexpr int kDialects = 32;
constexpr int kBins = 256;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// (p, q, r) of the shapes, the ramp, square and cube weights (sum 8), one
// nibble per shape (shape 0 in the low nibble): (8,0,0) (6,2,0) (4,4,0)
// (3,5,0) (2,5,1) (0,8,0) (1,3,4) (0,3,5).  Held in registers, not in a
// local-memory table.
constexpr uint32_t kShapeP = 0x01023468u, kShapeQ = 0x33855420u, kShapeR = 0x54010000u;

__host__ __device__ constexpr int shape_coef(int s, int k) {
  return static_cast<int>(((k == 0 ? kShapeP : (k == 1 ? kShapeQ : kShapeR)) >> (4 * s)) & 15u);
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

// Qerror is at most 16129 (< 2^14), so two dialects share a word and four
// entries sum without carrying across the halves.  qerr2[b][w] holds
// Qerror[2w][b] | Qerror[2w + 1][b] << 16 for w < 16 and again at w + 16, so
// the two half-warps, scoring different blocks, read disjoint banks.
struct Tables {
  uint32_t qerr2[kBins][32];
  uint8_t qval[kDialects][kBins];
  int lvl[kDialects][8];  // the formatbook L[d][i]
};

// Fills the tables; ends with a __syncthreads.
__device__ void build_tables(Tables* tb) {
  for (int idx = threadIdx.x; idx < kDialects * 8; idx += blockDim.x)
    tb->lvl[idx / 8][idx % 8] = level(idx / 8, idx % 8);
  __syncthreads();
  for (int idx = threadIdx.x; idx < kDialects * kBins; idx += blockDim.x) {
    const int d = idx / kBins, b = idx % kBins;
    uint32_t best = 0xFFFFFFFFu;
    int bi = 0;
    for (int i = 0; i < 8; ++i) {
      const int diff = 2 * b + 1 - 32 * tb->lvl[d][i];
      const uint32_t sq = static_cast<uint32_t>(diff * diff);
      if (sq < best) {
        best = sq;
        bi = i;
      }
    }
    uint16_t* row = reinterpret_cast<uint16_t*>(tb->qerr2[b]);
    row[d] = static_cast<uint16_t>(best);       // word d / 2, half d % 2
    row[32 + d] = static_cast<uint16_t>(best);  // the copy for the upper half-warp
    tb->qval[d][b] = static_cast<uint8_t>(bi);
  }
  __syncthreads();
}

// e4m3 encoding of L/8, 0 <= L <= 15 (normal for L >= 1: exponent field
// p + 4 with p = floor(log2 L), mantissa (L - 2^p) 2^(3-p)).
__host__ __device__ constexpr uint32_t e4m3_eighths(int L) {
  return L == 0 ? 0u
                : static_cast<uint32_t>(
                      (((L >= 8 ? 3 : L >= 4 ? 2 : L >= 2 ? 1 : 0) + 4) << 3) |
                      ((L - (1 << (L >= 8 ? 3 : L >= 4 ? 2 : L >= 2 ? 1 : 0)))
                       << (3 - (L >= 8 ? 3 : L >= 4 ? 2 : L >= 2 ? 1 : 0))));
}

// Eight codes (element k in nibble k) -> eight e4m3 bytes.  E: the dialect's
// magnitudes e4m3(L_i/8), byte i of the pair (lo, hi); `prmt` picks byte i for
// each code's level index, and the code's sign bit (nibble bit 3) moves to
// bit 7 of its byte.
__device__ __forceinline__ uint2 decode8_e4m3(uint32_t w, uint2 E) {
  const uint32_t v03 = __byte_perm(E.x, E.y, w & 0x7777u);
  const uint32_t v47 = __byte_perm(E.x, E.y, (w >> 16) & 0x7777u);
  const uint32_t s = w & 0x88888888u;
  const uint32_t t03 = __byte_perm(s, 0u, 0x1100u);  // bytes s0 s0 s1 s1
  const uint32_t t47 = __byte_perm(s, 0u, 0x3322u);  // bytes s2 s2 s3 s3
  const uint32_t s03 = ((t03 << 4) & 0x00800080u) | (t03 & 0x80008000u);
  const uint32_t s47 = ((t47 << 4) & 0x00800080u) | (t47 & 0x80008000u);
  return make_uint2(v03 | s03, v47 | s47);
}

// Byte i of the pair (lo, hi): e4m3(L[d][i] / 8) of dialect d.
__device__ __forceinline__ uint2 e4m3_levels(int d) {
  uint32_t lo = 0, hi = 0;
  for (int i = 0; i < 4; ++i) {
    lo |= e4m3_eighths(level(d, i)) << (8 * i);
    hi |= e4m3_eighths(level(d, i + 4)) << (8 * i);
  }
  return make_uint2(lo, hi);
}

// 2^n as binary32 for n in [-127, 127] (n = -127: the subnormal 2^-127).
__device__ __forceinline__ float pow2f(int n) {
  return n >= -126 ? __int_as_float((n + 127) << 23) : __int_as_float(0x00400000);
}

// One warp quantises 8 blocks (256 consecutive elements of a row): lane l
// holds elements 8l .. 8l + 7 in a[] (block l / 4).  Returns the lane's 8 codes
// (element k in nibble k) and sets e and d of the lane's block.  `bins` is the
// warp's 8 x 32 byte scratch.
__device__ __forceinline__ uint32_t quant_warp_chunk(const float (&a)[8], const Tables& tb,
                                                     uint8_t (*bins_sm)[kBlock], int lane, int& e_out,
                                                     int& d_out) {
  const int blk = lane >> 2;
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
  *reinterpret_cast<uint2*>(&bins_sm[blk][8 * (lane & 3)]) =
      make_uint2(bins[0] | (bins[1] << 8) | (bins[2] << 16) | (static_cast<uint32_t>(bins[3]) << 24),
                 bins[4] | (bins[5] << 8) | (bins[6] << 16) | (static_cast<uint32_t>(bins[7]) << 24));
  __syncwarp();
  // dialect choice, two blocks at a time: half-warp h scores block 2jj + h,
  // lane w of it dialects 2w and 2w + 1 (one packed table read per bin);
  // the block's 32 bins come as two broadcast 16-byte reads
  int my_d = 0;
  const int half = lane >> 4, w = lane & 15;
#pragma unroll 2
  for (int jj = 0; jj < 4; ++jj) {
    const int j = 2 * jj + half;
    const uint4 q0 = *reinterpret_cast<const uint4*>(&bins_sm[j][0]);
    const uint4 q1 = *reinterpret_cast<const uint4*>(&bins_sm[j][16]);
    const uint32_t bw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int k4 = 0; k4 < 8; ++k4) {
      uint32_t p = 0;  // four entries, both halves below 2^16
#pragma unroll
      for (int k = 0; k < 4; ++k) p += tb.qerr2[(bw[k4] >> (8 * k)) & 0xFFu][lane];
      lo += p & 0xFFFFu;
      hi += p >> 16;
    }
    uint32_t key = min((lo << 5) | static_cast<uint32_t>(2 * w),
                       (hi << 5) | static_cast<uint32_t>(2 * w + 1));
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) key = min(key, __shfl_xor_sync(0xffffffffu, key, off));
    const uint32_t k_even = __shfl_sync(0xffffffffu, key, 0);
    const uint32_t k_odd = __shfl_sync(0xffffffffu, key, 16);
    if (blk == 2 * jj) my_d = static_cast<int>(k_even & 31u);
    if (blk == 2 * jj + 1) my_d = static_cast<int>(k_odd & 31u);
  }
  uint32_t packed = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t code = (a[k] < 0.f ? 8u : 0u) | tb.qval[my_d][bins[k]];
    packed |= code << (4 * k);
  }
  __syncwarp();  // the scratch is rewritten by the next chunk
  e_out = e;
  d_out = my_d;
  return packed;
}

__device__ __forceinline__ void load_chunk8(const uint16_t* __restrict__ src, int lane,
                                            float (&a)[8]) {
  const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src) + lane);
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    a[2 * k] = __uint_as_float(w[k] << 16);
    a[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint16_t block_word(int e, int d) {
  return static_cast<uint16_t>((static_cast<uint32_t>(e) & 0xFFu) |
                               (static_cast<uint32_t>(d) << 8));
}

// --------------------------------------------------------------------------
// SD4 quantiser with the dialect choice on the tensor cores.  A block's cost
// for dialect d, sum_k Qerror[d][b_k], equals sum_b count[b] Qerror[d][b]
// with count the block's histogram over the 256 bins: an exact integer
// product of the count matrix (128 blocks x 256 bins, unsigned bytes, at most
// 32) with the cost table split into low and high bytes (64 x 256 unsigned
// bytes: Qerror <= 16129 = 63 * 256 + 1), accumulated in int32 (at most
// 32 * 255 per column: exact).  One thread per block: it loads the block,
// takes e and the bins, builds its row of the count matrix in shared memory
// (zeroed, then one non-returning shared add per element into a byte
// counter), and after the MMA reads its row of the costs back from tensor
// memory, takes the argmin (smallest d on ties) and writes the codes.
namespace tc {

constexpr int kTileBlocks = 128;  // rows of the count matrix per tile
constexpr int kThreads = kTileBlocks;
constexpr int kHHalf = kTileBlocks * 128;  // one K-half of the count matrix (128 bins)
constexpr int kQHalf = 64 * 128;           // one K-half of the cost bytes (64 rows)
constexpr int kOffH = 0;
constexpr int kOffQ = kOffH + 2 * kHHalf;
constexpr int kOffE4 = kOffQ + 2 * kQHalf;
constexpr int kOffLvl = kOffE4 + kDialects * 8;
constexpr int kOffMisc = kOffLvl + kDialects * 8 * 4;  // mbarrier, TMEM address, abort flag
constexpr int kSmemBytes = kOffMisc + 16 + 1024;       // + alignment slack
constexpr int kTmemCols = 64;
static_assert(kOffQ % 1024 == 0, "alignment");

// Byte offset of (row r, byte c < 128) in a K-major tile of 128-byte rows
// stored with the 128-byte swizzle.
__device__ __forceinline__ int sw128(int r, int c) {
  return r * 128 + ((((c >> 4) ^ (r & 7)) << 4) | (c & 15));
}

// Instruction descriptor: kind::i8 with unsigned A and B, int32 D, K-major.
__host__ __device__ constexpr uint32_t idesc_u8(int M, int N) {
  return (2u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

template <bool E4M3>
__global__ void __launch_bounds__(kThreads) sd4_quant_tc_kernel(const uint16_t* __restrict__ x,
                                                               int64_t rows, int K,
                                                               uint8_t* __restrict__ out,
                                                               uint16_t* __restrict__ meta) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  uint8_t* sp = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  uint8_t* H = sp + kOffH;
  uint8_t* Q = sp + kOffQ;
  uint2* e4 = reinterpret_cast<uint2*>(sp + kOffE4);
  int* lvl = reinterpret_cast<int*>(sp + kOffLvl);
  const uint32_t bar = sbase + kOffMisc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sp + kOffMisc + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sp + kOffMisc + 12);
  const int tid = threadIdx.x, warp = tid >> 5;

  for (int i = tid; i < kDialects * 8; i += kThreads) lvl[i] = level(i / 8, i % 8);
  __syncthreads();
  for (int idx = tid; idx < kDialects * kBins; idx += kThreads) {
    const int d = idx / kBins, b = idx % kBins;
    uint32_t best = 0xFFFFFFFFu;
    for (int i = 0; i < 8; ++i) {
      const int diff = 2 * b + 1 - 32 * lvl[d * 8 + i];
      best = min(best, static_cast<uint32_t>(diff * diff));
    }
    uint8_t* qh = Q + (b >> 7) * kQHalf;
    qh[sw128(d, b & 127)] = static_cast<uint8_t>(best & 0xFFu);      // low bytes: rows 0..31
    qh[sw128(32 + d, b & 127)] = static_cast<uint8_t>(best >> 8);    // high bytes: rows 32..63
  }
  for (int d = tid; d < kDialects; d += kThreads) {
    uint32_t lo = 0, hi = 0;
    for (int i = 0; i < 4; ++i) {
      lo |= e4m3_eighths(lvl[d * 8 + i]) << (8 * i);
      hi |= e4m3_eighths(lvl[d * 8 + i + 4]) << (8 * i);
    }
    e4[d] = make_uint2(lo, hi);
  }
  fence_proxy_async_smem();  // the cost bytes are read by the tensor cores
  if (tid == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int64_t nblocks = rows * static_cast<int64_t>(K / kBlock);
  const int64_t ntiles = (nblocks + kTileBlocks - 1) / kTileBlocks;
  uint32_t phase = 0;
  uint8_t* hrow0 = H + tid * 128;
  uint8_t* hrow1 = H + kHHalf + tid * 128;
  // the block's 32 elements (blocks are consecutive: row-major, K % 32 == 0);
  // the next tile's are loaded while this one is processed
  auto load_block = [&](int64_t tt, uint4 (&r)[4]) {
    const int64_t bb = tt * kTileBlocks + tid;
    const uint4* src = reinterpret_cast<const uint4*>(x + bb * kBlock);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      r[q] = (tt < ntiles && bb < nblocks) ? __ldcs(src + q) : make_uint4(0u, 0u, 0u, 0u);
  };
  uint4 nxt[4];
  load_block(blockIdx.x, nxt);
  for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x) {
    const int64_t blk = t * kTileBlocks + tid;
    const bool valid = blk < nblocks;
    uint4 raw4[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) raw4[q] = nxt[q];
    load_block(t + gridDim.x, nxt);
    float amax = 0.f;
    uint32_t neg = 0;  // bit k: element k is negative
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t w[4] = {raw4[q].x, raw4[q].y, raw4[q].z, raw4[q].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float a0 = __uint_as_float(w[k] << 16), a1 = __uint_as_float(w[k] & 0xFFFF0000u);
        amax = fmaxf(amax, fmaxf(fabsf(a0), fabsf(a1)));
        neg |= (a0 < 0.f ? 1u : 0u) << (8 * q + 2 * k);
        neg |= (a1 < 0.f ? 1u : 0u) << (8 * q + 2 * k + 1);
      }
    }
    int e = 0;
    if (amax != 0.f) {
      const int ef = (__float_as_uint(amax) >> 23) & 0xFF;
      e = ef == 0 ? -126 : max(ef - 127, -126);
    }
    const float sc = pow2f(-e);  // exact; |x| 2^-e < 2
    uint32_t binw[8];            // bins, 4 per word, element k in byte k % 4 of word k / 4
    // this block's row of the count matrix: zero, then one add per element
    // chunk order rotated by the row: the 8 lanes of a store phase hit 8
    // different 16-byte bank groups (rows are 128 bytes apart)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      reinterpret_cast<uint4*>(hrow0)[c ^ (tid & 7)] = make_uint4(0u, 0u, 0u, 0u);
      reinterpret_cast<uint4*>(hrow1)[c ^ (tid & 7)] = make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t w[4] = {raw4[q].x, raw4[q].y, raw4[q].z, raw4[q].w};
      uint32_t bw0 = 0, bw1 = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t h = (k & 1) ? (w[k >> 1] & 0xFFFF0000u) : (w[k >> 1] << 16);
        const float v = __fmul_rn(__fmul_rn(fabsf(__uint_as_float(h)), sc), 128.f);
        const int bv = static_cast<int>(v);  // truncation = floor for v >= 0
        const uint32_t b = static_cast<uint32_t>(bv > 255 ? 255 : bv);
        if (k < 4)
          bw0 |= b << (8 * k);
        else
          bw1 |= b << (8 * (k - 4));
        const int off = (b >> 7) * kHHalf + sw128(tid, static_cast<int>(b & 127u));
        atomicAdd(reinterpret_cast<uint32_t*>(H + (off & ~3)), 1u << (8 * (off & 3)));
      }
      binw[2 * q] = bw0;
      binw[2 * q + 1] = bw1;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_u8(kTileBlocks, 64);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int half = j >> 2, koff = (j & 3) * 32;
        mma_i8(tmem_base, smem_desc_sw128(sbase + kOffH + half * kHHalf + koff),
               smem_desc_sw128(sbase + kOffQ + half * kQHalf + koff), idesc, j != 0);
      }
      mma_commit(bar);
      if (!mbar_wait_bounded(bar, phase, abort_flag, kErrWaitMma)) *abort_flag = 1;
      tc_fence_before();
    }
    __syncthreads();
    if (*abort_flag) break;  // uniform: every thread sees the flag after the barrier
    phase ^= 1u;
    tc_fence_after();
    uint32_t lo[32], hi[32];
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * warp) << 16);
    tmem_ld_32x32b_x32(taddr, lo);
    tmem_ld_32x32b_x32(taddr + 32, hi);
    tmem_wait_ld();
    uint32_t best = 0xFFFFFFFFu;
    int d = 0;
#pragma unroll
    for (int dd = 0; dd < kDialects; ++dd) {
      const uint32_t cost = hi[dd] * 256u + lo[dd];
      if (cost < best) {
        best = cost;
        d = dd;
      }
    }
    // Qvalue[d][b], the nearest level, is the number of level midpoints
    // 16 (L_i + L_i+1) below 2b + 1 (odd against even: never a tie).  As
    // 2b + 1 > 16 s  <=>  b >= 8 s  <=>  (b >> 3) >= s, it depends on b >> 3
    // (0..31) alone: the block's dialect gives the count for all 32 values
    // as three bit planes (bit v of P_j = bit j of the count at b >> 3 = v),
    // summed from the seven masks {v >= s_i} by a bit-sliced counter.
    uint32_t P0 = 0, P1 = 0, P2 = 0;
#pragma unroll
    for (int i = 0; i < 7; ++i) {
      const int si = lvl[d * 8 + i] + lvl[d * 8 + i + 1];  // 0..30
      const uint32_t m = si >= 32 ? 0u : (0xFFFFFFFFu << si);
      const uint32_t c0 = P0 & m;
      P0 ^= m;
      const uint32_t c1 = P1 & c0;
      P1 ^= c0;
      P2 ^= c1;  // the count is at most 7
    }
    uint32_t cw[4];  // codes, element k in nibble k % 8 of word k / 8
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t c = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t v = (binw[(8 * q + k) >> 2] >> (8 * (k & 3) + 3)) & 31u;  // b >> 3
        const uint32_t idx =
            ((P0 >> v) & 1u) | (((P1 >> v) & 1u) << 1) | (((P2 >> v) & 1u) << 2);
        const uint32_t code = (((neg >> (8 * q + k)) & 1u) << 3) | idx;
        c |= code << (4 * k);
      }
      cw[q] = c;
    }
    if (valid) {
      if (E4M3) {
        const uint2 E = e4[d];
        const uint2 o0 = decode8_e4m3(cw[0], E), o1 = decode8_e4m3(cw[1], E);
        const uint2 o2 = decode8_e4m3(cw[2], E), o3 = decode8_e4m3(cw[3], E);
        uint4* dst = reinterpret_cast<uint4*>(out + blk * kBlock);
        dst[0] = make_uint4(o0.x, o0.y, o1.x, o1.y);
        dst[1] = make_uint4(o2.x, o2.y, o3.x, o3.y);
      } else {
        *reinterpret_cast<uint4*>(out + blk * (kBlock / 2)) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
      }
      meta[blk] = block_word(e, d);
    }
    tc_fence_before();  // this tile's tensor-memory reads precede the next MMA
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    const unsigned long long t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 2000000ull) __nanosleep(1000);
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace tc

// Activation decomposition of the salient rows (SemanticDialect "Resumen
// técnico" §2.B): output row i holds 2K codes, those of x[rows[i]] followed by
// those of the residual Delta = x - x_hat, and 2K/32 block words.  x_hat =
// (-1)^s L/8 2^e is exact in binary32 (e >= -126 keeps L 2^(e-3) a multiple
// of 2^-149) and so is the difference: an element rounded to a nonzero level
// has |x| >= 2^(e-4), both are multiples of 2^(e-11) and |Delta| < 2^(e+2);
// one rounded to level 0 has Delta = x.  An index outside [0, M) gives zero
// codes and words for the row and sets kErrIndex.
__global__ void __launch_bounds__(kThreads) sd4_decomp_kernel(
    const uint16_t* __restrict__ x, int64_t M, int K, const int32_t* __restrict__ rows, int64_t S,
    uint8_t* __restrict__ codes2, uint16_t* __restrict__ meta2) {
  __shared__ Tables tb;
  __shared__ __align__(16) uint8_t s_bins[kWarps][8][kBlock];
  build_tables(&tb);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blk = lane >> 2;
  const int64_t chunks_per_row = K / 256;
  const int64_t num_chunks = S * chunks_per_row;
  for (int64_t c = static_cast<int64_t>(blockIdx.x) * kWarps + warp; c < num_chunks;
       c += static_cast<int64_t>(gridDim.x) * kWarps) {
    const int64_t i = c / chunks_per_row;
    const int col0 = static_cast<int>(c % chunks_per_row) * 256;
    uint8_t* crow = codes2 + i * static_cast<int64_t>(K);        // 2K codes
    uint16_t* mrow = meta2 + i * static_cast<int64_t>(K / 16);   // 2K/32 words
    const int64_t r = rows[i];
    if (r < 0 || r >= M) {
      *reinterpret_cast<uint32_t*>(crow + col0 / 2 + 4 * lane) = 0u;
      *reinterpret_cast<uint32_t*>(crow + K / 2 + col0 / 2 + 4 * lane) = 0u;
      if ((lane & 3) == 0) {
        mrow[col0 / kBlock + blk] = 0;
        mrow[K / kBlock + col0 / kBlock + blk] = 0;
      }
      if (lane == 0) atomicOr(&g_error_word, kErrIndex);
      continue;
    }
    float a[8];
    load_chunk8(x + r * static_cast<int64_t>(K) + col0, lane, a);
    int e, d;
    const uint32_t pa = quant_warp_chunk(a, tb, s_bins[warp], lane, e, d);
    *reinterpret_cast<uint32_t*>(crow + col0 / 2 + 4 * lane) = pa;
    if ((lane & 3) == 0) mrow[col0 / kBlock + blk] = block_word(e, d);
    const float sc = pow2f(e);
    float delta[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t code = (pa >> (4 * k)) & 15u;
      const float xh = __fmul_rn(static_cast<float>(tb.lvl[d][code & 7u]) * 0.125f, sc);
      delta[k] = __fsub_rn(a[k], (code & 8u) ? -xh : xh);
    }
    int e2, d2;
    const uint32_t pd = quant_warp_chunk(delta, tb, s_bins[warp], lane, e2, d2);
    *reinterpret_cast<uint32_t*>(crow + K / 2 + col0 / 2 + 4 * lane) = pd;
    if ((lane & 3) == 0) mrow[K / kBlock + col0 / kBlock + blk] = block_word(e2, d2);
  }
}

// --------------------------------------------------------------------------
// SD4 layer GEMM: out[m][n] = bf16(fl(sum_k x_hat[m][k] w_hat[n][k]) + bias[n])
// with x_hat, w_hat the decoded SD4 values.  The decoded values are exact in
// bf16, so the product runs on the tensor cores as a bf16 GEMM
// (tcgen05.mma.kind::f16, binary32 accumulators in tensor memory): codes come
// by TMA, 12 warps decode them into the 128-byte-swizzled operand tiles.
//
// Persistent, one CTA per SM, tiles of 128 x 256, 64 K elements per stage.
// Warp roles: 0 TMA producer (codes every stage, block words every 4 stages:
// a TMA row is at least 16 bytes = 8 block words = 256 elements); 1 TMEM
// allocation and the MMA issuer; 2-5 epilogue; 6-17 decode.
// --------------------------------------------------------------------------

namespace gemm_sd4 {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int kOpStages = 3, kPkStages = 3, kMetaSlots = 2;
constexpr int kEpiWarps = 4, kDecWarps = 12;
constexpr int kThreads = 32 * (2 + kEpiWarps + kDecWarps);
constexpr int kOpA = BM * BK * 2, kOpB = BN * BK * 2, kOpStage = kOpA + kOpB;  // bf16 tiles
constexpr int kPkA = BM * BK / 2, kPkB = BN * BK / 2;                          // code tiles
constexpr int kMetaA = BM * 16, kMetaB = BN * 16;                              // 8 words/row
constexpr int kNumBars = 2 * kPkStages + 2 * kMetaSlots + 2 * kOpStages + 4;
constexpr int kTmemCols = 2 * BN;

// WDEC: the weights come already decoded (bf16, by qs_sd4_decode) and go by
// TMA straight into their operand tile; only the activation rows are decoded.
template <bool WDEC>
struct SCfg {
  static constexpr int kDecRows = WDEC ? BM : BM + BN;  // operand rows decoded per stage
  static constexpr int kPkStage = WDEC ? kPkA : kPkA + kPkB;
  static constexpr int kMetaSlot = WDEC ? kMetaA : kMetaA + kMetaB;
  static constexpr int kOffOp = 0;
  static constexpr int kOffPk = kOffOp + kOpStages * kOpStage;
  static constexpr int kOffMeta = kOffPk + kPkStages * kPkStage;
  static constexpr int kOffBar = kOffMeta + kMetaSlots * kMetaSlot;
  static constexpr int kOffEpi = (kOffBar + 8 * kNumBars + 15) / 16 * 16;  // bias of a tile
  static constexpr int kOffPair = kOffEpi + BN * 4;                          // pair table
  static constexpr int kOffMisc = kOffPair + kDialects * 256 * 4;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  // arrivals completing an operand stage: the decode warps, plus the
  // producer's arm of the weight tile's TMA bytes
  static constexpr int kOpFullCount = kDecWarps + (WDEC ? 1 : 0);
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
};

__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4)                                // D format: F32
         | (1u << 7)                              // A: BF16
         | (1u << 10)                             // B: BF16
         | (static_cast<uint32_t>(N >> 3) << 17)  // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24); // M / 16
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

struct Bars {
  uint32_t base;
  __device__ uint32_t at(int i) const { return base + 8u * i; }
  __device__ uint32_t pk_full(int s) const { return at(s); }
  __device__ uint32_t pk_empty(int s) const { return at(kPkStages + s); }
  __device__ uint32_t meta_full(int s) const { return at(2 * kPkStages + s); }
  __device__ uint32_t meta_empty(int s) const { return at(2 * kPkStages + kMetaSlots + s); }
  __device__ uint32_t op_full(int s) const { return at(2 * kPkStages + 2 * kMetaSlots + s); }
  __device__ uint32_t op_empty(int s) const {
    return at(2 * kPkStages + 2 * kMetaSlots + kOpStages + s);
  }
  __device__ uint32_t acc_full(int b) const {
    return at(2 * kPkStages + 2 * kMetaSlots + 2 * kOpStages + b);
  }
  __device__ uint32_t acc_empty(int b) const {
    return at(2 * kPkStages + 2 * kMetaSlots + 2 * kOpStages + 2 + b);
  }
};

// Decodes 16 codes (8 bytes) of one block into 16 bf16 values (two 16-byte
// chunks).  Fast path: the pair table holds, for each dialect and code byte,
// the two signed magnitudes L/8 as a bf16 pair; one bf16x2 multiply by 2^e
// scales both exactly (a power of two, the result normal for e >= -123).
// Blocks below that (results near the subnormal range) take the binary32 path.
__device__ __forceinline__ void decode16_float(uint2 c, int e, const uint32_t* T, uint4& lo,
                                               uint4& hi);

__device__ __forceinline__ void decode16(uint2 c, uint32_t word, const uint32_t* pairs,
                                         uint4& lo, uint4& hi) {
  const int e = static_cast<int8_t>(word & 0xFFu);
  const int d = static_cast<int>(word >> 8) & 31;
  const uint32_t* T = pairs + 256 * d;
  if (e < -123) {
    decode16_float(c, e, T, lo, hi);
    return;
  }
  const uint32_t sbits = static_cast<uint32_t>(e + 127) << 7;  // bf16 2^e
  const uint32_t s2 = sbits | (sbits << 16);
  const __nv_bfloat162 scale = *reinterpret_cast<const __nv_bfloat162*>(&s2);
  uint32_t out[8];
  const uint32_t cw[2] = {c.x, c.y};
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t v = T[(cw[h] >> (8 * k)) & 0xFFu];
      const __nv_bfloat162 r = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&v), scale);
      out[4 * h + k] = *reinterpret_cast<const uint32_t*>(&r);
    }
  lo = make_uint4(out[0], out[1], out[2], out[3]);
  hi = make_uint4(out[4], out[5], out[6], out[7]);
}

__device__ __forceinline__ void decode16_float(uint2 c, int e, const uint32_t* T, uint4& lo,
                                               uint4& hi) {
  // T[code] (a byte whose high nibble is 0) holds the signed L/8 of `code` as bf16
  const float sc = pow2f(e);
  uint32_t out[8];
  const uint32_t cw[2] = {c.x, c.y};
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t c0 = (cw[h] >> (8 * k)) & 0xFu, c1 = (cw[h] >> (8 * k + 4)) & 0xFu;
      const float v0 = __fmul_rn(__uint_as_float(T[c0] << 16), sc);
      const float v1 = __fmul_rn(__uint_as_float(T[c1] << 16), sc);
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(v0, v1);
      out[4 * h + k] = *reinterpret_cast<const uint32_t*>(&b2);
    }
  lo = make_uint4(out[0], out[1], out[2], out[3]);
  hi = make_uint4(out[4], out[5], out[6], out[7]);
}

template <bool WDEC>
__global__ void __launch_bounds__(kThreads, 1)
    sd4_gemm_kernel(const __grid_constant__ CUtensorMap tmCA, const __grid_constant__ CUtensorMap tmCB,
                    const __grid_constant__ CUtensorMap tmMA, const __grid_constant__ CUtensorMap tmMB,
                    const __grid_constant__ CUtensorMap tmWB, const uint16_t* __restrict__ bias,
                    uint16_t* __restrict__ out, int M, int N, int K, int kb_wrap,
                    const int32_t* __restrict__ out_rows, int out_M) {
  using C = SCfg<WDEC>;
  constexpr int kOffOp = C::kOffOp, kOffPk = C::kOffPk, kOffMeta = C::kOffMeta;
  constexpr int kOffBar = C::kOffBar, kOffEpi = C::kOffEpi, kOffPair = C::kOffPair;
  constexpr int kOffMisc = C::kOffMisc, kPkStage = C::kPkStage, kMetaSlot = C::kMetaSlot;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  uint8_t* sp = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  Bars bars{sbase + kOffBar};
  float* epi_b = reinterpret_cast<float*>(sp + kOffEpi);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sp + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sp + kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (N + BN - 1) / BN;
  const int num_tiles = ((M + BM - 1) / BM) * n_tiles;
  const int kblocks = K / BK;

  uint32_t* pairs = reinterpret_cast<uint32_t*>(sp + kOffPair);
  for (int i = threadIdx.x; i < kDialects * 256; i += blockDim.x) {
    const int d = i / 256, b = i % 256;
    uint32_t h[2];
    for (int j = 0; j < 2; ++j) {
      const int code = (b >> (4 * j)) & 15;
      // L/8 is exact in bf16: the binary32 value's top 16 bits
      const float v = static_cast<float>(level(d, code & 7)) * 0.125f;
      h[j] = (__float_as_uint(v) >> 16) | ((code & 8) ? 0x8000u : 0u);
    }
    pairs[i] = h[0] | (h[1] << 16);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPkStages; ++s) {
      mbar_init(bars.pk_full(s), 1);
      mbar_init(bars.pk_empty(s), kDecWarps);
    }
    for (int s = 0; s < kMetaSlots; ++s) {
      mbar_init(bars.meta_full(s), 1);
      mbar_init(bars.meta_empty(s), kDecWarps);
    }
    for (int s = 0; s < kOpStages; ++s) {
      mbar_init(bars.op_full(s), C::kOpFullCount);
      mbar_init(bars.op_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bars.acc_full(b), 1);
      mbar_init(bars.acc_empty(b), kEpiWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {  // producer
      int s = 0, ms = 0, so = 0;
      uint32_t ph = 0, mph = 0, pho = 0;
      for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
        const int m0 = (t / n_tiles) * BM, n0 = (t % n_tiles) * BN;
        for (int kb = 0, kbw = 0; kb < kblocks; ++kb, kbw = (kbw + 1 == kb_wrap ? 0 : kbw + 1)) {
          // kbw: the weights' K-block (the A rows may be longer: [x | Delta]
          // against [w | w]); kb_wrap % 4 == 0 keeps the block words aligned
          if ((kb & 3) == 0) {
            if (!mbar_wait_bounded(bars.meta_empty(ms), mph ^ 1u, abort_flag, kErrWaitProducer))
              break;
            const uint32_t dst = sbase + kOffMeta + ms * kMetaSlot;
            mbar_arrive_expect_tx(bars.meta_full(ms), kMetaSlot);
            tma_load_2d(dst, &tmMA, (kb / 4) * 16, m0, bars.meta_full(ms));
            if (!WDEC) tma_load_2d(dst + kMetaA, &tmMB, (kbw / 4) * 16, n0, bars.meta_full(ms));
            if (++ms == kMetaSlots) { ms = 0; mph ^= 1u; }
          }
          if (!mbar_wait_bounded(bars.pk_empty(s), ph ^ 1u, abort_flag, kErrWaitProducer)) break;
          const uint32_t dst = sbase + kOffPk + s * kPkStage;
          mbar_arrive_expect_tx(bars.pk_full(s), kPkStage);
          tma_load_2d(dst, &tmCA, kb * (BK / 2), m0, bars.pk_full(s));
          if (!WDEC) tma_load_2d(dst + kPkA, &tmCB, kbw * (BK / 2), n0, bars.pk_full(s));
          if (++s == kPkStages) { s = 0; ph ^= 1u; }
          if (WDEC) {  // decoded weights: TMA into the operand stage's B tile
            if (!mbar_wait_bounded(bars.op_empty(so), pho ^ 1u, abort_flag, kErrWaitProducer))
              break;
            const uint32_t ob = sbase + kOffOp + so * kOpStage + kOpA;
            mbar_arrive_expect_tx(bars.op_full(so), kOpB);
            tma_load_2d(ob, &tmWB, kbw * BK, n0, bars.op_full(so));
            if (++so == kOpStages) { so = 0; pho ^= 1u; }
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      constexpr uint32_t idesc = idesc_bf16(BM, BN);
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
        const int buf = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait_bounded(bars.acc_empty(buf), aph ^ 1u, abort_flag, kErrWaitMma)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(buf * BN);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_bounded(bars.op_full(s), ph, abort_flag, kErrWaitMma)) break;
          tc_fence_after();
          const uint32_t a0 = sbase + kOffOp + s * kOpStage;
          const uint32_t b0 = a0 + kOpA;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_bf16(d, smem_desc_sw128(a0 + kk * 32), smem_desc_sw128(b0 + kk * 32), idesc,
                     (kb | kk) != 0);
          mma_commit(bars.op_empty(s));
          if (++s == kOpStages) { s = 0; ph ^= 1u; }
        }
        mma_commit(bars.acc_full(buf));
      }
    }
  } else if (warp < 2 + kEpiWarps) {  // epilogue: TMEM lanes 32 * (warp & 3) ..
    const int quad = warp & 3;
    const int et = threadIdx.x - 64;
    int it = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
      const int buf = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      const int m0 = (t / n_tiles) * BM, n0 = (t % n_tiles) * BN;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      for (int i = et; i < BN; i += 128) {
        const int n = n0 + i;
        epi_b[i] = (n < N && bias) ? __uint_as_float(static_cast<uint32_t>(bias[n]) << 16) : 0.f;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (!mbar_wait_bounded(bars.acc_full(buf), aph, abort_flag, kErrWaitEpilogue)) break;
      tc_fence_after();
      const int row = m0 + 32 * quad + lane;
      int orow = row < M ? row : -1;  // the output row this accumulator row goes to
      if (out_rows && orow >= 0) {
        orow = out_rows[row];
        if (orow < 0 || orow >= out_M) {
          atomicOr(&g_error_word, kErrIndex);
          orow = -1;
        }
      }
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * quad) << 16) +
                             static_cast<uint32_t>(buf * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(taddr + 32 * c, r);
        tmem_wait_ld();
        const int n = n0 + 32 * c;
        if (orow >= 0 && n < N) {
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float y0 = __fadd_rn(__uint_as_float(r[2 * j]), epi_b[32 * c + 2 * j]);
            const float y1 = __fadd_rn(__uint_as_float(r[2 * j + 1]), epi_b[32 * c + 2 * j + 1]);
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(y0, y1);
            pk[j] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          uint16_t* dst = out + static_cast<int64_t>(orow) * N + n;
#pragma unroll
          for (int v = 0; v < 4; ++v)
            if (n + 8 * v + 8 <= N)
              *reinterpret_cast<uint4*>(dst + 8 * v) =
                  make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.acc_empty(buf));
    }
  } else {  // decode warps
    const int dt = threadIdx.x - 32 * (2 + kEpiWarps);  // 0 .. 32 kDecWarps - 1
    int s = 0, so = 0, ms = 0;
    uint32_t ph = 0, pho = 0, mph = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      for (int kb = 0; kb < kblocks; ++kb) {
        if ((kb & 3) == 0 &&
            !mbar_wait_bounded(bars.meta_full(ms), mph, abort_flag, kErrWaitUnpack))
          break;
        if (!mbar_wait_bounded(bars.pk_full(s), ph, abort_flag, kErrWaitUnpack)) break;
        if (!mbar_wait_bounded(bars.op_empty(so), pho ^ 1u, abort_flag, kErrWaitUnpack)) break;
        const uint8_t* pk = sp + kOffPk + s * kPkStage;
        const uint8_t* mt = sp + kOffMeta + ms * kMetaSlot;
        uint8_t* op = sp + kOffOp + so * kOpStage;
        // tasks: (operand row r in 0..383, 16-element chunk c in 0..3)
#pragma unroll
        for (int j = 0; j < (C::kDecRows * 4 + 32 * kDecWarps - 1) / (32 * kDecWarps); ++j) {
          const int task = dt + 32 * kDecWarps * j;
          if (task >= C::kDecRows * 4) break;
          const int r = task >> 2, c = task & 3;
          const uint2 codes = *reinterpret_cast<const uint2*>(pk + r * (BK / 2) + c * 8);
          // block word: block (kb % 4) * 2 + c / 2 of this row's 8-word slot row
          const uint16_t word = *reinterpret_cast<const uint16_t*>(
              mt + r * 16 + ((kb & 3) * 2 + (c >> 1)) * 2);
          uint4 lo, hi;
          decode16(codes, word, pairs, lo, hi);
          uint8_t* rowp = op + r * 128;  // x rows 0..127, then W rows (operand B at +kOpA)
          *reinterpret_cast<uint4*>(rowp + (((2 * c) ^ (r & 7)) << 4)) = lo;
          *reinterpret_cast<uint4*>(rowp + (((2 * c + 1) ^ (r & 7)) << 4)) = hi;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bars.op_full(so));
          mbar_arrive(bars.pk_empty(s));
          if ((kb & 3) == 3) mbar_arrive(bars.meta_empty(ms));
        }
        if (++s == kPkStages) { s = 0; ph ^= 1u; }
        if (++so == kOpStages) { so = 0; pho ^= 1u; }
        if ((kb & 3) == 3 && ++ms == kMetaSlots) { ms = 0; mph ^= 1u; }
      }
    }
    // drain: the MMA's last releases of the operand stages have landed
    if (lane == 0)
      for (int i = 0; i < kOpStages; ++i) {
        if (!mbar_wait_bounded(bars.op_empty(so), pho ^ 1u, abort_flag, kErrWaitUnpack)) break;
        if (++so == kOpStages) { so = 0; pho ^= 1u; }
      }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    const unsigned long long t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 2000000ull) __nanosleep(1000);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// Decoded values of an SD4 matrix, bf16 [rows, K]: one thread per 16 elements
// (8 code bytes and the block word) through the same pair table.
__global__ void __launch_bounds__(256) sd4_decode_kernel(const uint8_t* __restrict__ codes,
                                                         const uint16_t* __restrict__ meta,
                                                         int64_t rows, int K,
                                                         uint16_t* __restrict__ out) {
  __shared__ uint32_t pairs[kDialects * 256];
  for (int i = threadIdx.x; i < kDialects * 256; i += blockDim.x) {
    const int d = i / 256, b = i % 256;
    uint32_t h[2];
    for (int j = 0; j < 2; ++j) {
      const int code = (b >> (4 * j)) & 15;
      const float v = static_cast<float>(level(d, code & 7)) * 0.125f;
      h[j] = (__float_as_uint(v) >> 16) | ((code & 8) ? 0x8000u : 0u);
    }
    pairs[i] = h[0] | (h[1] << 16);
  }
  __syncthreads();
  const int64_t per_row = K / 16;
  const int64_t n = rows * per_row;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < n;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = t / per_row;
    const int c = static_cast<int>(t % per_row);  // 16-element chunk of the row
    const uint2 cw = *reinterpret_cast<const uint2*>(codes + row * (K / 2) + c * 8);
    const uint32_t word = meta[row * (K / 32) + c / 2];
    uint4 lo, hi;
    decode16(cw, word, pairs, lo, hi);
    uint4* dst = reinterpret_cast<uint4*>(out + row * static_cast<int64_t>(K) + c * 16);
    dst[0] = lo;
    dst[1] = hi;
  }
}

}  // namespace gemm_sd4

}  // namespace sd4
}  // namespace qs
