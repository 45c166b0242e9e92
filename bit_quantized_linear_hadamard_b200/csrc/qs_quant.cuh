// Fused rotate -> online scale -> quantize -> pack kernels.
//
// DVD-Quant, "Resumen técnico" §2.B (ARQ): a Hadamard rotation spreads the
// extreme values across channels, and the quantization factors are computed
// at run time from the rotated values.  Serves both the per-token activation
// quantization (alpha = clip ratio) and the offline per-output-channel weight
// quantization (alpha = 1, scale multiplied by the exact 2^-7 that carries the
// two 1/sqrt(128) normalisations).
//
// Per row: u = block Walsh-Hadamard transform of the bf16 row (binary32
// butterfly, stages h = 1, 2, 4, ..., 64 in that order), t = fl(alpha*amax),
// s = fl(t/qmax) (stored), inv = fl(qmax/t), q = clamp(rint(fl(u*inv))) with
// rows of t < 2^-120 treated as zero rows.
//
// Two kernels compute exactly that:
//  * rotate_quant_half_kernel (K <= 16384): half a 128-element Hadamard block
//    per thread, stages h = 1..32 in registers (packed f32x2 arithmetic), stage
//    64 with the partner thread; a CTA holds whole rows (double-buffered in
//    shared memory) and reduces their absmax through shared memory.
//  * rotate_quant_group_kernel (longer rows): 8 elements per thread, stages
//    h = 1, 2, 4 in registers and h = 8..64 by xor-shuffles, one row per CTA.
// Rounding to the nearest integer, ties to even, is done by adding 1.5*2^23:
// for |r| < 2^22 the sum is exactly representable only at integers, so the IEEE
// round-to-nearest-even addition performs the rounding and the integer lands in
// the low mantissa bits (two's complement in the low byte).
#pragma once

#include "qs_ptx.cuh"

namespace qs {

constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr float kZeroRowT = 0x1p-120f;

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

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

// Per-row factors from the row absmax: s (dequantization, stored) and inv
// (quantization multiplier); both 0 for a zero row.
template <int QMAX>
__device__ __forceinline__ void row_factors(float amax, float alpha, float& s, float& inv) {
  const float t = __fmul_rn(alpha, amax);
  if (t >= kZeroRowT) {
    s = __fdiv_rn(t, static_cast<float>(QMAX));
    inv = __fdiv_rn(static_cast<float>(QMAX), t);
  } else {
    s = 0.f;
    inv = 0.f;
  }
}

// Bits of fl(clamp(fl(u*inv)) + 1.5*2^23): the low byte is the two's complement
// code rint_half_even(clamp(fl(u*inv))) (clamping to integer bounds commutes
// with rounding, so this equals clamp(rint(fl(u*inv)))).
template <int QMAX>
__device__ __forceinline__ uint32_t code_bits(float u, float inv) {
  float r = __fmul_rn(u, inv);
  r = fminf(fmaxf(r, -static_cast<float>(QMAX)), static_cast<float>(QMAX));
  return __float_as_uint(__fadd_rn(r, kRoundMagic));
}

// 8 codes (low byte/nibble of c[0..7]) -> packed bytes.
__device__ __forceinline__ uint32_t pack8_int4(const uint32_t (&c)[8]) {
  uint32_t b[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) b[m] = ((c[2 * m + 1] << 4) & 0xF0u) | (c[2 * m] & 0x0Fu);
  return __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
}

__device__ __forceinline__ uint32_t pack4_int8(uint32_t c0, uint32_t c1, uint32_t c2,
                                               uint32_t c3) {
  return __byte_perm(__byte_perm(c0, c1, 0x0040), __byte_perm(c2, c3, 0x0040), 0x5410);
}

// --------------------------------------------------------------------------
// Rows of up to 128 Hadamard blocks: half a block per thread.
//
// A persistent CTA walks groups of `rpc` consecutive rows.  A group is one
// contiguous span of x; it is copied into shared memory by coalesced 16-byte
// cp.async, two groups in flight (double buffer).  Chunk i (16 bytes) of block
// tb of the group (block b of row r, tb = r * nblk + b) is stored at chunk
// i ^ (tb & 15), which keeps the copy free of bank conflicts.
//
// Threads 2tb and 2tb+1 own the low and high 64 elements of block tb.  A half
// lives in registers as 32 pairs (v[j], v[j + 32]): butterfly stages h = 1..16
// pair (j, j + h) and (j + 32, j + 32 + h) alike, so two butterflies are one
// packed add.rn.f32x2 and one sub.rn.f32x2 (independent IEEE binary32
// operations); stage 32 works inside the pairs; stage 64 pairs the two threads:
// each takes its partner's value p by an xor-shuffle and forms fl(p + sg * own)
// with sg = +1 (low half: a + b) or -1 (high half: a - b) in one packed
// fma.rn.f32x2 -- sg * own is exact, so the single rounding is that of the
// butterfly's add or subtract.
// --------------------------------------------------------------------------

__device__ __forceinline__ uint64_t pack_f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void unpack_f2(uint64_t p, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p));
}

__device__ __forceinline__ uint64_t add_f2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint64_t sub_f2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint64_t mul_f2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint64_t fma_f2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ void cp_async_wait_1() {
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}

// Copies the rows of group g (those below `rows`) into a shared-memory stage.
__device__ __forceinline__ void copy_group(const uint16_t* __restrict__ x, int64_t rows, int K,
                                           int rpc, int64_t g, uint32_t stage) {
  const int64_t row0 = g * rpc;
  int64_t nrows = rows - row0;
  if (nrows > rpc) nrows = rpc;
  const int chunks = static_cast<int>(nrows) * (K / 8);  // 16-byte chunks
  const char* src = reinterpret_cast<const char*>(x + row0 * static_cast<int64_t>(K));
  for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
    const int tb = c >> 4, i = c & 15;
    cp_async16(stage + tb * 256 + ((i ^ (tb & 15)) << 4), src + static_cast<int64_t>(c) * 16);
  }
}

template <int BITS>
__global__ void __launch_bounds__(256) rotate_quant_half_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int K, int nblk, int rpc, int64_t num_groups,
    float alpha, float scale_mul, int rotate, uint8_t* __restrict__ out,
    float* __restrict__ scale_out) {
  constexpr int kQmax = BITS == 4 ? 7 : 127;
  constexpr int kOutBytes = 64 * BITS / 8;  // packed bytes per half block
  extern __shared__ __align__(16) uint8_t qsmem[];
  __shared__ unsigned int row_amax[2][128];

  const int tid = threadIdx.x;
  const int tb = tid >> 1;       // block within the group
  const int up = tid & 1;        // which half of the block
  const int rl = tb / nblk;
  const int blk = tb - rl * nblk;
  const bool worker = rl < rpc;
  const int stage_bytes = rpc * K * 2;
  const uint32_t stage0 = smem_u32(qsmem);
  const uint64_t sg2 = pack_f2(up ? -1.f : 1.f, up ? -1.f : 1.f);

  if (tid < rpc) row_amax[0][tid] = 0u;
  copy_group(x, rows, K, rpc, blockIdx.x, stage0);
  cp_async_commit();

  int it = 0;
  for (int64_t g = blockIdx.x; g < num_groups; g += gridDim.x, ++it) {
    const int par = it & 1;
    const int64_t gn = g + gridDim.x;
    if (gn < num_groups) copy_group(x, rows, K, rpc, gn, stage0 + (par ^ 1) * stage_bytes);
    cp_async_commit();
    cp_async_wait_1();
    __syncthreads();  // the current stage is complete; row_amax[par ^ 1] is free
    if (tid < rpc) row_amax[par ^ 1][tid] = 0u;

    const int64_t row = g * rpc + rl;
    const bool active = worker && row < rows;
    uint64_t p[32];  // (v[j], v[j + 32]) of this half block
    if (active) {
      const uint8_t* blkp = qsmem + par * stage_bytes + tb * 256;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c0 = 8 * up + i, c1 = 8 * up + i + 4;
        const uint4 lo = *reinterpret_cast<const uint4*>(blkp + ((c0 ^ (tb & 15)) << 4));
        const uint4 hi = *reinterpret_cast<const uint4*>(blkp + ((c1 ^ (tb & 15)) << 4));
        const uint32_t lw[4] = {lo.x, lo.y, lo.z, lo.w};
        const uint32_t hw[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float a0, a1, b0, b1;
          bf16x2_to_f32(lw[k], a0, a1);
          bf16x2_to_f32(hw[k], b0, b1);
          p[8 * i + 2 * k] = pack_f2(a0, b0);
          p[8 * i + 2 * k + 1] = pack_f2(a1, b1);
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) p[j] = 0ull;
    }

    if (rotate) {
#pragma unroll
      for (int h = 1; h < 32; h <<= 1)
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if ((j & h) == 0) {
            const uint64_t a = p[j], b = p[j + h];
            p[j] = add_f2(a, b);
            p[j + h] = sub_f2(a, b);
          }
#pragma unroll
      for (int j = 0; j < 32; ++j) {  // h = 32: (v[j], v[j + 32])
        float a, b;
        unpack_f2(p[j], a, b);
        p[j] = pack_f2(__fadd_rn(a, b), __fsub_rn(a, b));
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) {  // h = 64: the partner thread holds the other half
        float a, b;
        unpack_f2(p[j], a, b);
        const float pa = __shfl_xor_sync(0xffffffffu, a, 1);
        const float pb = __shfl_xor_sync(0xffffffffu, b, 1);
        p[j] = fma_f2(sg2, p[j], pack_f2(pa, pb));
      }
    }

    float m[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) m[k] = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float a, b;
      unpack_f2(p[j], a, b);
      m[j & 3] = fmaxf(m[j & 3], fmaxf(fabsf(a), fabsf(b)));
    }
    float amax = fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    // non-negative binary32 values order like their bit patterns
    if (active && up == 0) atomicMax(&row_amax[par][rl], __float_as_uint(amax));
    __syncthreads();  // row maxima complete; every thread is done reading the stage
    if (!active) continue;

    float s, inv;
    row_factors<kQmax>(__uint_as_float(row_amax[par][rl]), alpha, s, inv);
    if (blk == 0 && up == 0) scale_out[row] = __fmul_rn(s, scale_mul);

    const uint64_t inv2 = pack_f2(inv, inv);
    const uint64_t magic2 = pack_f2(kRoundMagic, kRoundMagic);
    uint32_t c[64];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float a, b;
      unpack_f2(mul_f2(p[j], inv2), a, b);
      a = fminf(fmaxf(a, -static_cast<float>(kQmax)), static_cast<float>(kQmax));
      b = fminf(fmaxf(b, -static_cast<float>(kQmax)), static_cast<float>(kQmax));
      float ca, cb;
      unpack_f2(add_f2(pack_f2(a, b), magic2), ca, cb);
      c[j] = __float_as_uint(ca);
      c[j + 32] = __float_as_uint(cb);
    }
    uint8_t* dst =
        out + row * static_cast<int64_t>(K * BITS / 8) + blk * (2 * kOutBytes) + up * kOutBytes;
    if (BITS == 4) {
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int e = 32 * q + 8 * k;
          const uint32_t cc[8] = {c[e], c[e + 1], c[e + 2], c[e + 3],
                                  c[e + 4], c[e + 5], c[e + 6], c[e + 7]};
          w[k] = pack8_int4(cc);
        }
        *reinterpret_cast<uint4*>(dst + 16 * q) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int e = 16 * q + 4 * k;
          w[k] = pack4_int8(c[e], c[e + 1], c[e + 2], c[e + 3]);
        }
        *reinterpret_cast<uint4*>(dst + 16 * q) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
}

// --------------------------------------------------------------------------
// Long rows: groups of 8 elements, shuffle stages, one row per CTA.
// Thread t of T owns groups t, t+T, ..., t+(G-1)T (a warp reads 512 contiguous
// bytes per load); the 16 groups of one Hadamard block sit in 16 consecutive
// lanes (T is a multiple of 32), so stage h = 8, 16, 32, 64 pairs lanes at
// xor-distance 1, 2, 4, 8.
// --------------------------------------------------------------------------
template <int G, int BITS, int MAXT>
__global__ void __launch_bounds__(MAXT) rotate_quant_group_kernel(const uint16_t* __restrict__ x,
                                                                  int K, float alpha,
                                                                  float scale_mul, int rotate,
                                                                  uint8_t* __restrict__ out,
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
#pragma unroll
      for (int h = 1; h < 8; h <<= 1)
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if ((e & h) == 0) butterfly(v[j][e], v[j][e + h]);
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

  float s, inv;
  row_factors<kQmax>(amax, alpha, s, inv);
  if (tid == 0) scale_out[row] = __fmul_rn(s, scale_mul);

#pragma unroll
  for (int j = 0; j < G; ++j) {
    const int g = tid + j * T;
    if (g >= ngroups) continue;
    uint32_t c[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) c[e] = code_bits<kQmax>(v[j][e], inv);
    if (BITS == 4) {
      *reinterpret_cast<uint32_t*>(out + row * static_cast<int64_t>(K >> 1) + g * 4) =
          pack8_int4(c);
    } else {
      *reinterpret_cast<uint2*>(out + row * static_cast<int64_t>(K) + g * 8) =
          make_uint2(pack4_int8(c[0], c[1], c[2], c[3]), pack4_int8(c[4], c[5], c[6], c[7]));
    }
  }
}

// Chooses (G groups per thread, T threads) for a row of `ngroups` 8-element
// groups: G <= 8, T a multiple of 32 and at most `max_t`, least idle slots,
// then the largest G.  Returns false if the row does not fit one pass.
inline bool choose_group_shape(int ngroups, int max_t, int* G_out, int* T_out) {
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

// Rows per CTA for the half-block kernel: 2*nblk threads per row, at most 256
// threads, fewest idle threads (blockDim is a multiple of 32), then the blockDim
// closest to 128.
inline int choose_rows_per_cta(int nblk) {
  int best = 1, best_waste = 1 << 30, best_dist = 1 << 30;
  for (int r = 1; r * 2 * nblk <= 256; ++r) {
    const int used = r * 2 * nblk;
    const int bd = (used + 31) / 32 * 32;
    const int waste = bd - used;
    const int dist = bd > 128 ? bd - 128 : 128 - bd;
    if (waste < best_waste || (waste == best_waste && dist < best_dist)) {
      best = r;
      best_waste = waste;
      best_dist = dist;
    }
  }
  return best;
}

template <int BITS>
inline cudaError_t launch_rotate_quant_bits(const uint16_t* x, int64_t rows, int K, float alpha,
                                            float scale_mul, int rotate, uint8_t* out,
                                            float* scale, cudaStream_t stream) {
  const int nblk = K / 128;
  if (nblk <= 128) {
    const int rpc = choose_rows_per_cta(nblk);
    const int threads = (rpc * 2 * nblk + 31) / 32 * 32;
    const int64_t groups = (rows + rpc - 1) / rpc;
    const int smem = 2 * rpc * K * 2;  // two stages of rpc rows
    auto kern = rotate_quant_half_kernel<BITS>;
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0, dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem)) !=
        cudaSuccess)
      return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    int64_t grid = static_cast<int64_t>(sms) * per_sm;
    if (grid > groups) grid = groups;
    kern<<<static_cast<unsigned>(grid), threads, smem, stream>>>(
        x, rows, K, nblk, rpc, groups, alpha, scale_mul, rotate, out, scale);
    return cudaGetLastError();
  }
  // Rows up to 2048 groups run with at most 256 threads so each thread keeps
  // its 8*G values in registers; longer rows use up to 1024.
  const int ngroups = K / 8;
  const bool wide = ngroups > 256 * 8;
  int G = 0, T = 0;
  if (!choose_group_shape(ngroups, wide ? 1024 : 256, &G, &T)) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(rows)), block(T);
#define QS_QUANT_CASE(GG)                                                                   \
  case GG:                                                                                  \
    if (wide)                                                                               \
      rotate_quant_group_kernel<GG, BITS, 1024>                                             \
          <<<grid, block, 0, stream>>>(x, K, alpha, scale_mul, rotate, out, scale);         \
    else                                                                                    \
      rotate_quant_group_kernel<GG, BITS, 256>                                              \
          <<<grid, block, 0, stream>>>(x, K, alpha, scale_mul, rotate, out, scale);         \
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
