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
// s = fl(t/qmax) (stored), inv = fl(qmax/t), q = clamp(rint(u*inv)) with the
// product exact and rounded once, and rows of t < 2^-120 treated as zero rows.
//
// Two kernels compute exactly that:
//  * rotate_quant_tma_kernel (K <= 16384): half a 128-element Hadamard block
//    per thread, stages h = 1..32 in registers (packed f32x2 arithmetic), stage
//    64 with the partner thread; row groups stream into a multi-stage
//    shared-memory ring by TMA; the row absmax is reduced through shared memory.
//  * rotate_quant_group_kernel (longer rows): 8 elements per thread, stages
//    h = 1, 2, 4 in registers and h = 8..64 by xor-shuffles, one row per CTA.
// Rounding to the nearest integer, ties to even, is one fused multiply-add
// fl(u*inv + 1.5*2^23): for |u*inv| < 2^22 (alpha >= 2^-14) the sum lies in
// [2^23, 2^24), where binary32 holds exactly the integers, so the single
// round-to-nearest-even of the exact u*inv + 1.5*2^23 is 1.5*2^23 +
// rint_half_even(u*inv) (1.5*2^23 is even), and the integer lands in the low
// mantissa bits (two's complement in the low 16 bits).
//
// Code widths: 4 bits (qmax 7, two codes per byte), 6 bits (qmax 31, the
// W4A6 activations of DVD-Quant, one int8 byte per code) and 8 bits (qmax 127).
#pragma once

#include "qs_host.cuh"
#include "qs_ptx.cuh"

namespace qs {

// Largest code magnitude of a b-bit symmetric grid, 2^(b-1) - 1.
__host__ __device__ constexpr int code_qmax(int bits) { return (1 << (bits - 1)) - 1; }
// Bits of storage per code: 4-bit codes are packed in nibbles, wider codes
// take one byte.
__host__ __device__ constexpr int code_storage_bits(int bits) { return bits == 4 ? 4 : 8; }

constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
// Depth of the activation kernel's shared-memory ring (rows of up to 128
// Hadamard blocks): two stages measured faster than three or four, which cost
// resident CTAs (the kernel is latency-bound and more warps per SM win).
constexpr int kQuantStages = 2;
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

// Bits of clamp(fl(u*inv + 1.5*2^23), 1.5*2^23 -+ qmax): the low byte is the
// two's complement code clamp(rint_half_even(u*inv), -qmax, qmax).
template <int QMAX>
__device__ __forceinline__ uint32_t code_bits(float u, float inv) {
  const float f = __fmaf_rn(u, inv, kRoundMagic);
  return __float_as_uint(fminf(fmaxf(f, kRoundMagic - static_cast<float>(QMAX)),
                               kRoundMagic + static_cast<float>(QMAX)));
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

// Clamping and packing of 8 codes on packed 16-bit lanes.  Input: bits of
// fl(u*inv + 1.5*2^23) without a clamp; their low 16 bits are the unclamped
// code q as int16 whenever |q| < 2^15, which holds for alpha >= 1/256
// (|q| <= qmax/alpha + 1 <= 32513).
__device__ __forceinline__ uint32_t s16x2_clamp(uint32_t w, uint32_t hi, uint32_t lo) {
  uint32_t r;
  asm("min.s16x2 %0, %1, %2;" : "=r"(r) : "r"(w), "r"(hi));
  asm("max.s16x2 %0, %1, %2;" : "=r"(r) : "r"(r), "r"(lo));
  return r;
}

// Clamped codes c[4h..4h+3] as 4 int8 bytes (h = 0 or 1).
template <int QMAX>
__device__ __forceinline__ uint32_t simd_bytes4(const uint32_t (&c)[8], int h) {
  constexpr uint32_t hi = (static_cast<uint32_t>(QMAX) << 16) | static_cast<uint32_t>(QMAX);
  constexpr uint32_t lo = ((0x10000u - QMAX) << 16) | (0x10000u - QMAX);
  const uint32_t w01 = s16x2_clamp(__byte_perm(c[4 * h], c[4 * h + 1], 0x5410), hi, lo);
  const uint32_t w23 = s16x2_clamp(__byte_perm(c[4 * h + 2], c[4 * h + 3], 0x5410), hi, lo);
  return __byte_perm(w01, w23, 0x6420);
}

// Clamped codes c[0..7] as 8 int4 nibbles (element 2j in the low nibble of
// byte j): the even and the odd codes are clamped as int16 pairs and narrowed
// to bytes separately, then one bit-select joins the even bytes' low nibbles
// with the odd bytes' low nibbles shifted up (16 instructions per 8 codes,
// where narrowing consecutive codes and merging adjacent bytes took 21).
__device__ __forceinline__ uint32_t simd_nibbles8(const uint32_t (&c)[8]) {
  constexpr uint32_t hi = (7u << 16) | 7u;
  constexpr uint32_t lo = ((0x10000u - 7u) << 16) | (0x10000u - 7u);
  const uint32_t e01 = s16x2_clamp(__byte_perm(c[0], c[2], 0x5410), hi, lo);
  const uint32_t e23 = s16x2_clamp(__byte_perm(c[4], c[6], 0x5410), hi, lo);
  const uint32_t o01 = s16x2_clamp(__byte_perm(c[1], c[3], 0x5410), hi, lo);
  const uint32_t o23 = s16x2_clamp(__byte_perm(c[5], c[7], 0x5410), hi, lo);
  const uint32_t ev = __byte_perm(e01, e23, 0x6420);  // bytes: c0 c2 c4 c6
  const uint32_t od = __byte_perm(o01, o23, 0x6420);  // bytes: c1 c3 c5 c7
  return (ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u);
}

// Sum of the signed codes held in packed words: 8 nibbles per word (4-bit) or
// 4 bytes per word.  Nibbles are moved to the high half of a byte (16 q, exact)
// and summed with dp4a, so the total is 16 x the code sum.
template <int STORE, int NW>
__device__ __forceinline__ int packed_code_sum(const uint32_t (&w)[NW]) {
  int acc = 0;
#pragma unroll
  for (int i = 0; i < NW; ++i) {
    if (STORE == 4) {
      acc = __dp4a(static_cast<int>((w[i] << 4) & 0xF0F0F0F0u), 0x01010101, acc);
      acc = __dp4a(static_cast<int>(w[i] & 0xF0F0F0F0u), 0x01010101, acc);
    } else {
      acc = __dp4a(static_cast<int>(w[i]), 0x01010101, acc);
    }
  }
  return STORE == 4 ? acc >> 4 : acc;
}

// Adds a per-thread code sum to rowsum[row]: the threads of one row that run
// together add within the warp first, their lowest lane does the atomic.
__device__ __forceinline__ void add_row_sum(int* rowsum, int64_t row, int part, int row_key) {
  const unsigned act = __activemask();
  const unsigned same = __match_any_sync(act, row_key);
  const int tot = __reduce_add_sync(same, part);
  if ((threadIdx.x & 31) == __ffs(same) - 1) atomicAdd(rowsum + row, tot);
}

// --------------------------------------------------------------------------
// Rows of up to 128 Hadamard blocks: half a block per thread.
//
// A persistent CTA walks groups of `rpc` consecutive rows.  A group is one
// contiguous span of x, viewed as rows of 64 bf16 (128 bytes); thread 0 loads
// it with one 2-D TMA copy (128-byte swizzle) into a stage of a `stages`-deep
// shared-memory ring and the copy completes on that stage's mbarrier, so the
// next groups are in flight while the current one is computed.
//
// Threads 2tb and 2tb+1 own the low and high 64 elements of block tb of the
// group = 128-byte row R = 2tb + up of the stage, whose 16-byte chunk i sits at
// chunk i ^ (R & 7): eight consecutive threads read eight different chunk
// positions, free of bank conflicts.  A half lives in registers as 32 pairs
// (v[j], v[j + 32]): butterfly stages h = 1..16 pair (j, j + h) and
// (j + 32, j + 32 + h) alike, so two butterflies are one packed add.rn.f32x2
// and one packed fma (independent IEEE binary32 operations; a - b is
// fma(b, -1, a): the product is exact, the one rounding is the subtraction's).
// Stage 32 works inside the pairs, as fma(b, c, a) with c = +-1; the high
// thread keeps its result swapped, (out[96 + j], out[64 + j]).  Stage 64 pairs
// the two threads, and each finishes both outputs of half the butterflies:
// it receives its partner's .y by one xor-shuffle (r) and forms
// (keep + r, keep - r) from its own .x (keep), giving (out[j], out[64 + j])
// in the low thread and (out[32 + j], -out[96 + j]) in the high one -- one
// shuffle per pair of values, where exchanging whole halves takes two.  The
// sign is exact and is undone by the quantisation multiplier of that lane.
//
// One __syncthreads per group: the row absmax (pair shuffle, then a
// shared-memory atomicMax of the bit patterns, triple-buffered so that no
// second barrier is needed) is complete after it, and every thread has read the
// stage, which thread 0 then refills.
// --------------------------------------------------------------------------

// Launch modes of the activation kernel: the plain hot path; gated on a
// device-side width (δ-GBS: returns at once unless *gate == gate_want); or
// also adding every row's code sum to rowsum[row] (zeroed by the caller).
// Separate instantiations keep the plain path free of either.
enum QuantMode { kPlain = 0, kGated = 1, kRowsum = 2 };

// BITS: code width (qmax 2^(BITS-1) - 1); STORE: storage per code, 4 (two
// codes per byte) or 8 (one byte per code, also for 4-bit codes).
template <int BITS, int STORE, bool SIMD_CLAMP, int MODE>
__global__ void __launch_bounds__(256) rotate_quant_tma_kernel(
    const __grid_constant__ CUtensorMap tmx, int64_t rows, int K, int nblk, int rpc,
    int64_t num_groups, int stages, float alpha, float scale_mul, int rotate,
    uint8_t* __restrict__ out, float* __restrict__ scale_out, const int* gate, int gate_want,
    int* __restrict__ rowsum) {
  if (MODE == kGated && *gate != gate_want) return;
  constexpr int kQmax = code_qmax(BITS);
  constexpr int kOutBytes = 64 * STORE / 8;  // packed bytes per half block
  extern __shared__ __align__(1024) uint8_t qsmem_raw[];
  __shared__ unsigned int row_amax[3][128];
  __shared__ int abort_flag;

  const uint32_t raw = smem_u32(qsmem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  uint8_t* base = qsmem_raw + pad;
  const uint32_t sbase = raw + pad;
  const int stage_bytes = rpc * K * 2;                    // one group = the TMA box
  const int stage_stride = (stage_bytes + 1023) / 1024 * 1024;
  const uint32_t bars = sbase + stages * stage_stride;    // full[s] mbarriers
  const int box_rows = rpc * K / 64;

  const int tid = threadIdx.x;
  const int tb = tid >> 1;  // block within the group
  const int up = tid & 1;   // which half of the block
  const int rl = tb / nblk;
  const int blk = tb - rl * nblk;
  const bool worker = rl < rpc;
  if (tid == 0) {
    for (int i = 0; i < stages; ++i) mbar_init(bars + 8 * i, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < rpc) row_amax[0][tid] = 0u;
  __syncthreads();
  if (tid == 0) {
    tma_prefetch_desc(&tmx);
    for (int i = 0; i < stages; ++i) {
      const int64_t g = blockIdx.x + static_cast<int64_t>(i) * gridDim.x;
      if (g >= num_groups) break;
      mbar_arrive_expect_tx(bars + 8 * i, stage_bytes);
      tma_load_2d(sbase + i * stage_stride, &tmx, 0, static_cast<int>(g * box_rows), bars + 8 * i);
    }
  }

  // Stage, phase and row-maximum buffer of group number `it`.  The launcher
  // uses a ring of two stages.  The packed (two codes per byte) instantiation
  // advances them as counters, the others derive them from `it`: with
  // identical outputs, each form measured the faster one for its
  // instantiation (packed W4 at the Wan FFN shape 96.4 -> 94.4 us; the
  // byte-code and 8-bit ones 98.6 -> 106 us with counters).
  int it = 0;
  int s_ctr = 0, rb_ctr = 0;
  uint32_t ph_ctr = 0;
  for (int64_t g = blockIdx.x; g < num_groups; g += gridDim.x, ++it) {
    int s, rb;
    uint32_t ph;
    if constexpr (STORE == 4) {
      static_assert(kQuantStages == 2, "the counters below step a ring of two stages");
      s = s_ctr;
      ph = ph_ctr;
      rb = rb_ctr;
      ph_ctr ^= static_cast<uint32_t>(s_ctr);
      s_ctr ^= 1;
      rb_ctr = rb_ctr == 2 ? 0 : rb_ctr + 1;
      if (tid < rpc) row_amax[rb_ctr][tid] = 0u;  // last read two groups ago
    } else {
      s = it % stages;
      ph = static_cast<uint32_t>(it / stages) & 1u;
      rb = it % 3;
      if (tid < rpc) row_amax[(it + 1) % 3][tid] = 0u;  // last read two groups ago
    }
    mbar_wait_bounded(bars + 8 * s, ph, &abort_flag, kErrWaitTma);

    const int64_t row = g * rpc + rl;
    const bool active = worker && row < rows;
    float2 p[32];  // (v[j], v[j + 32]) of this half block
    if (active) {
      const int R = 2 * tb + up;
      const uint8_t* rowp = base + s * stage_stride + R * 128;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 lo = *reinterpret_cast<const uint4*>(rowp + ((i ^ (R & 7)) << 4));
        const uint4 hi = *reinterpret_cast<const uint4*>(rowp + (((i + 4) ^ (R & 7)) << 4));
        const uint32_t lw[4] = {lo.x, lo.y, lo.z, lo.w};
        const uint32_t hw[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float a0, a1, b0, b1;
          bf16x2_to_f32(lw[k], a0, a1);
          bf16x2_to_f32(hw[k], b0, b1);
          p[8 * i + 2 * k] = make_float2(a0, b0);
          p[8 * i + 2 * k + 1] = make_float2(a1, b1);
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) p[j] = make_float2(0.f, 0.f);
    }

    if (rotate) {
      const float2 neg1 = make_float2(-1.f, -1.f);
#pragma unroll
      for (int h = 1; h < 32; h <<= 1)
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if ((j & h) == 0) {
            const float2 a = p[j], b = p[j + h];
            p[j] = __fadd2_rn(a, b);
            p[j + h] = __ffma2_rn(b, neg1, a);  // a - b, one rounding
          }
      // h = 32 inside the pairs (the high thread's result swapped)
      const float2 c32 = make_float2(up ? -1.f : 1.f, up ? 1.f : -1.f);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        p[j] = __ffma2_rn(make_float2(p[j].y, p[j].y), c32, make_float2(p[j].x, p[j].x));
      // h = 64: (keep + r, keep - r) with r the partner's .y
      const float2 pm = make_float2(1.f, -1.f);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float r = __shfl_xor_sync(0xffffffffu, p[j].y, 1);
        p[j] = __ffma2_rn(make_float2(r, r), pm, make_float2(p[j].x, p[j].x));
      }
    } else {
      // no rotation: the same element layout, low (j, 64 + j), high (32 + j, 96 + j)
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float r = __shfl_xor_sync(0xffffffffu, up ? p[j].x : p[j].y, 1);
        p[j] = up ? make_float2(r, p[j].y) : make_float2(p[j].x, r);
      }
    }

    float m[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) m[k] = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) m[j & 3] = fmaxf(m[j & 3], fmaxf(fabsf(p[j].x), fabsf(p[j].y)));
    float amax = fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    // non-negative binary32 values order like their bit patterns
    if (active && up == 0) atomicMax(&row_amax[rb][rl], __float_as_uint(amax));
    __syncthreads();  // row maxima complete; every thread has read stage s
    if (abort_flag) break;
    if (tid == 0) {
      const int64_t gn = g + static_cast<int64_t>(stages) * gridDim.x;
      if (gn < num_groups) {
        mbar_arrive_expect_tx(bars + 8 * s, stage_bytes);
        tma_load_2d(sbase + s * stage_stride, &tmx, 0, static_cast<int>(gn * box_rows),
                    bars + 8 * s);
      }
    }
    if (!active) continue;

    // every thread needs the multiplier; one thread per row stores the scale
    const float t_row = __fmul_rn(alpha, __uint_as_float(row_amax[rb][rl]));
    const bool zero_row = !(t_row >= kZeroRowT);
    const float inv = zero_row ? 0.f : __fdiv_rn(static_cast<float>(kQmax), t_row);
    if (blk == 0 && up == 0)
      scale_out[row] = zero_row ? 0.f : __fmul_rn(__fdiv_rn(t_row, static_cast<float>(kQmax)), scale_mul);

    // the high thread's .y holds -out[96 + j] after the rotation
    const float2 inv2 = make_float2(inv, (rotate && up) ? -inv : inv);
    const float2 magic2 = make_float2(kRoundMagic, kRoundMagic);
    [[maybe_unused]] constexpr float kQ = static_cast<float>(kQmax);
    // Codes of 8 consecutive pairs: .x = elements 32 up + 8k .. + 7 of the
    // block, .y = elements 64 + 32 up + 8k .. + 7.
    uint32_t wlo[STORE == 4 ? 4 : 8], whi[STORE == 4 ? 4 : 8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t clo[8], chi[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float2 cb = __ffma2_rn(p[8 * k + e], inv2, magic2);  // magic + rint(u * inv)
        if (!SIMD_CLAMP) {
          cb.x = fminf(fmaxf(cb.x, kRoundMagic - kQ), kRoundMagic + kQ);
          cb.y = fminf(fmaxf(cb.y, kRoundMagic - kQ), kRoundMagic + kQ);
        }
        clo[e] = __float_as_uint(cb.x);
        chi[e] = __float_as_uint(cb.y);
      }
      if (SIMD_CLAMP) {
        if (STORE == 4) {
          wlo[k] = simd_nibbles8(clo);
          whi[k] = simd_nibbles8(chi);
        } else {
          wlo[2 * k] = simd_bytes4<kQmax>(clo, 0);
          wlo[2 * k + 1] = simd_bytes4<kQmax>(clo, 1);
          whi[2 * k] = simd_bytes4<kQmax>(chi, 0);
          whi[2 * k + 1] = simd_bytes4<kQmax>(chi, 1);
        }
      } else if (STORE == 4) {
        wlo[k] = pack8_int4(clo);
        whi[k] = pack8_int4(chi);
      } else {
        wlo[2 * k] = pack4_int8(clo[0], clo[1], clo[2], clo[3]);
        wlo[2 * k + 1] = pack4_int8(clo[4], clo[5], clo[6], clo[7]);
        whi[2 * k] = pack4_int8(chi[0], chi[1], chi[2], chi[3]);
        whi[2 * k + 1] = pack4_int8(chi[4], chi[5], chi[6], chi[7]);
      }
    }
    // the .x codes cover elements 32 up .. 32 up + 31 of the block, the .y
    // codes 64 + 32 up .. 64 + 32 up + 31: two 16-byte aligned pieces
    uint8_t* dst = out + row * static_cast<int64_t>(K * STORE / 8) + blk * (2 * kOutBytes);
    uint8_t* dlo = dst + up * (kOutBytes / 2);
    uint8_t* dhi = dst + kOutBytes + up * (kOutBytes / 2);
    if (STORE == 4) {
      *reinterpret_cast<uint4*>(dlo) = make_uint4(wlo[0], wlo[1], wlo[2], wlo[3]);
      *reinterpret_cast<uint4*>(dhi) = make_uint4(whi[0], whi[1], whi[2], whi[3]);
    } else {
      *reinterpret_cast<uint4*>(dlo) = make_uint4(wlo[0], wlo[1], wlo[2], wlo[3]);
      *reinterpret_cast<uint4*>(dlo + 16) = make_uint4(wlo[4], wlo[5], wlo[6], wlo[7]);
      *reinterpret_cast<uint4*>(dhi) = make_uint4(whi[0], whi[1], whi[2], whi[3]);
      *reinterpret_cast<uint4*>(dhi + 16) = make_uint4(whi[4], whi[5], whi[6], whi[7]);
    }
    if (MODE == kRowsum)
      add_row_sum(rowsum, row, packed_code_sum<STORE>(wlo) + packed_code_sum<STORE>(whi), rl);
  }
  if (abort_flag) {
    // a wait gave up: let copies already in flight land before the CTA exits
    const unsigned long long t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 2000000ull) __nanosleep(1000);
  }
}

// --------------------------------------------------------------------------
// Long rows: groups of 8 elements, shuffle stages, one row per CTA.
// Thread t of T owns groups t, t+T, ..., t+(G-1)T (a warp reads 512 contiguous
// bytes per load); the 16 groups of one Hadamard block sit in 16 consecutive
// lanes (T is a multiple of 32), so stage h = 8, 16, 32, 64 pairs lanes at
// xor-distance 1, 2, 4, 8.
// --------------------------------------------------------------------------
template <int G, int BITS, int STORE, int MAXT>
__global__ void __launch_bounds__(MAXT) rotate_quant_group_kernel(const uint16_t* __restrict__ x,
                                                                  int K, float alpha,
                                                                  float scale_mul, int rotate,
                                                                  uint8_t* __restrict__ out,
                                                                  float* __restrict__ scale_out,
                                                                  const int* gate, int gate_want,
                                                                  int* __restrict__ rowsum) {
  if (gate != nullptr && *gate != gate_want) return;
  __shared__ int s_rowsum;
  if (threadIdx.x == 0) s_rowsum = 0;
  constexpr int kQmax = code_qmax(BITS);
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

  int rsum = 0;
#pragma unroll
  for (int j = 0; j < G; ++j) {
    const int g = tid + j * T;
    if (g >= ngroups) continue;
    uint32_t c[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) c[e] = code_bits<kQmax>(v[j][e], inv);
    if (STORE == 4) {
      const uint32_t pw[1] = {pack8_int4(c)};
      *reinterpret_cast<uint32_t*>(out + row * static_cast<int64_t>(K >> 1) + g * 4) = pw[0];
      if (rowsum) rsum += packed_code_sum<STORE>(pw);
    } else {
      const uint32_t pw[2] = {pack4_int8(c[0], c[1], c[2], c[3]), pack4_int8(c[4], c[5], c[6], c[7])};
      *reinterpret_cast<uint2*>(out + row * static_cast<int64_t>(K) + g * 8) =
          make_uint2(pw[0], pw[1]);
      if (rowsum) rsum += packed_code_sum<STORE>(pw);
    }
  }
  if (rowsum) {  // one row per CTA: block total, one store
    atomicAdd(&s_rowsum, rsum);
    __syncthreads();
    if (tid == 0) rowsum[row] = s_rowsum;
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

template <int BITS, int STORE>
// gate / gate_want: when gate is not null the kernels return at once unless
// *gate == gate_want (read on the device when they start).  rowsum: when not
// null, every row's code sum is added to rowsum[row] (zeroed by the caller).
inline cudaError_t launch_rotate_quant_bits(const uint16_t* x, int64_t rows, int K, float alpha,
                                            float scale_mul, int rotate, uint8_t* out,
                                            float* scale, cudaStream_t stream,
                                            const int* gate = nullptr, int gate_want = 0,
                                            int* rowsum = nullptr) {
  const int nblk = K / 128;
  const int rpc = nblk <= 128 ? choose_rows_per_cta(nblk) : 0;
  const int64_t groups = rpc ? (rows + rpc - 1) / rpc : 0;
  // TMA row coordinates are 32-bit: groups * (rpc * K / 64) must stay below 2^31
  if (nblk <= 128 && groups * (static_cast<int64_t>(rpc) * K / 64) < (int64_t{1} << 31)) {
    const int threads = (rpc * 2 * nblk + 31) / 32 * 32;
    const int stage_stride = (rpc * K * 2 + 1023) / 1024 * 1024;
    const int stages = kQuantStages;
    const int smem = stages * stage_stride + 8 * stages + 1024;
    CUtensorMap tmx;
    if (!make_tensor_map_2d(&tmx, x, 64, static_cast<uint64_t>(rows) * K / 64, 64, rpc * K / 64,
                            true, 2))
      return cudaErrorInvalidValue;
    // codes clamp on packed int16 lanes when the unclamped code fits int16
    const bool simd = alpha >= 1.0f / 256.0f;
    auto kern = simd ? rotate_quant_tma_kernel<BITS, STORE, true, kPlain>
                     : rotate_quant_tma_kernel<BITS, STORE, false, kPlain>;
    if (gate)
      kern = simd ? rotate_quant_tma_kernel<BITS, STORE, true, kGated>
                  : rotate_quant_tma_kernel<BITS, STORE, false, kGated>;
    else if (rowsum)
      kern = simd ? rotate_quant_tma_kernel<BITS, STORE, true, kRowsum>
                  : rotate_quant_tma_kernel<BITS, STORE, false, kRowsum>;
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem)) !=
        cudaSuccess)
      return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    int64_t grid = static_cast<int64_t>(sms) * per_sm;
    if (grid > groups) grid = groups;
    kern<<<static_cast<unsigned>(grid), threads, smem, stream>>>(
        tmx, rows, K, nblk, rpc, groups, stages, alpha, scale_mul, rotate, out, scale, gate,
        gate_want, rowsum);
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
      rotate_quant_group_kernel<GG, BITS, STORE, 1024>                                      \
          <<<grid, block, 0, stream>>>(x, K, alpha, scale_mul, rotate, out, scale, gate,     \
                                       gate_want, rowsum);                                  \
    else                                                                                    \
      rotate_quant_group_kernel<GG, BITS, STORE, 256>                                       \
          <<<grid, block, 0, stream>>>(x, K, alpha, scale_mul, rotate, out, scale, gate,     \
                                       gate_want, rowsum);                                  \
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
                                       cudaStream_t stream, const int* gate = nullptr,
                                       int gate_want = 0, int* rowsum = nullptr,
                                       bool byte_codes = false) {
  // byte_codes: 4-bit codes written one per byte (6- and 8-bit codes always are)
  switch (bits) {
    case 4:
      return byte_codes
                 ? launch_rotate_quant_bits<4, 8>(x, rows, K, alpha, scale_mul, rotate, out, scale,
                                                  stream, gate, gate_want, rowsum)
                 : launch_rotate_quant_bits<4, 4>(x, rows, K, alpha, scale_mul, rotate, out, scale,
                                                  stream, gate, gate_want, rowsum);
    case 6:
      return launch_rotate_quant_bits<6, 8>(x, rows, K, alpha, scale_mul, rotate, out, scale,
                                            stream, gate, gate_want, rowsum);
    case 8:
      return launch_rotate_quant_bits<8, 8>(x, rows, K, alpha, scale_mul, rotate, out, scale,
                                            stream, gate, gate_want, rowsum);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace qs
