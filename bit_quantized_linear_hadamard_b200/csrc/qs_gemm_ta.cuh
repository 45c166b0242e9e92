// W4A4 integer GEMM with the activation operand widened into tensor memory
// (tcgen05, sm_100a).
//
// The low-bit product of the rotated layer (DVD-Quant "Resumen técnico" §1 and
// §4, W4A4), both operands stored as packed 4-bit codes:
//   acc[m][n] = sum_k q_a[m][k] * q_w[n][k]                       (int32, exact)
//   out[m][n] = bf16(fl(fl(fl(s_a[m] * s_w[n]) * float(acc)) + bias[n]))
//
// tcgen05 has no 4-bit integer kind, so both operands are widened to int8.
// Widening through shared memory costs, per K-block and CTA, the TMA write of
// the packed tiles, their read, the write of the widened tiles and the tensor
// core's read of them; at the int8 MMA rate that shared-memory traffic, not
// the MMA, bounds the main loop.  Here the activation operand goes to TENSOR
// memory instead: tcgen05.mma may read A from tensor memory, so the widening
// warps store the widened activation rows with tcgen05.st (lane = token row,
// four K elements per 32-bit column) and only the weights take the
// shared-memory path.  Per K-block and CTA that is 52 KB of shared-memory
// traffic for 128 x 192 x 128 multiply-adds, against 96 KB for
// 128 x 256 x 128 when both operands are widened in shared memory.
//
// Structure: persistent clusters of two CTAs (one per SM of a TPC), output
// tiles of 256 x 192 (n fastest: the packed weight stays in L2), one
// tcgen05.mma.cta_group::2.kind::i8 (M = 256, N = 192, K = 32) per 32-deep K
// step issued by the leader CTA; CTA r holds rows [128r, 128r + 128) of the
// activation tile (in its tensor memory) and rows [96r, 96r + 96) of the
// weight tile (in its shared memory).  Tensor memory of each CTA: two 192-column
// int32 accumulators (the epilogue of one tile runs under the main loop of the
// next) and four 32-column activation stages = 512 columns.
//
// Widening (as in the shared-memory GEMM): each packed 16-byte chunk (32
// nibbles, K elements 32j .. 32j + 31) becomes 32 bytes, the even elements'
// nibbles in the high half of 16 bytes, then the odd elements'; the byte read
// as int8 is 16 q, the tensor core sums 256 acc, the epilogue shifts it back
// (exact).  Both operands use this K order (the activation's 32 bytes as eight
// consecutive tensor-memory columns, the weight's as two consecutive 16-byte
// chunks of the 128-byte swizzled row), so every dot product is unchanged.
//
// Warp roles (both CTAs; 14 warps):
//   warp 0       TMA producer (packed activation and weight tiles)
//   warp 1       TMEM allocation; leader: MMA issuer; other CTA: relay of
//                "this CTA's stage is widened" to the leader (16-byte bulk copy)
//   warps 2-5    epilogue (tcgen05.ld of this CTA's accumulator rows)
//   warps 6-9    activation widening into tensor memory, one token row per thread
//   warps 10-13  weight widening into the 128-byte-swizzled shared-memory tile
#pragma once

#include <cuda_bf16.h>

#include "qs.h"
#include "qs_gemm.cuh"
#include "qs_host.cuh"
#include "qs_ptx.cuh"

namespace qs {
namespace gemm_ta {

using gemm::epilogue_chunk;

constexpr int BM = 256;      // tile rows (tokens), 128 per CTA
constexpr int BN = 192;      // tile columns (output channels), 96 weight rows per CTA
constexpr int HM = 128;
constexpr int HN = 96;
constexpr int BK = 128;      // K elements per stage
constexpr int kStages = 4;
constexpr int kAccCols = BN;                 // one accumulator
constexpr int kACol0 = 2 * BN;               // first tensor-memory column of the activation ring
constexpr int kACols = BK / 4;               // columns per activation stage
constexpr int kTmemCols = 512;
static_assert(kACol0 + kStages * kACols <= kTmemCols, "tensor memory columns");
constexpr int kShift = 8;                    // both operands carry the factor 16

constexpr int kOpBytes = HN * BK;            // widened weight tile (shared memory)
constexpr int kPkA = HM * BK / 2;            // packed activation tile (64-byte swizzle)
constexpr int kPkB = HN * BK / 2;            // packed weight tile (plain rows)
constexpr int kPkStage = kPkA + kPkB;
constexpr int kOffOp = 0;
constexpr int kOffPk = kOffOp + kStages * kOpBytes;
constexpr int kOffBar = kOffPk + kStages * kPkStage;
// pk_full, pk_empty, op_empty, ready, op_full (x kStages), acc_full, acc_empty (x2)
constexpr int kNumBars = 5 * kStages + 4;
constexpr int kOffEpi = (kOffBar + 8 * kNumBars + 15) / 16 * 16;
constexpr int kOffMisc = kOffEpi + 3 * BN * 4;
constexpr int kOffSignal = kOffMisc + 16;
constexpr int kSmemBytes = kOffSignal + 16 * kStages + 1024;
static_assert(kOpBytes % 1024 == 0 && kPkStage % 1024 == 0 && kPkA % 1024 == 0, "alignment");
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");

constexpr int kEpiWarps = 4;
constexpr int kAWarps = 4;
constexpr int kBWarps = 4;
constexpr int kThreads = 32 * (2 + kEpiWarps + kAWarps + kBWarps);
constexpr int kWidenWarps = kAWarps + kBWarps;
constexpr int kBChunksPerThread = (kPkB / 16) / (32 * kBWarps);
static_assert((kPkB / 16) % (32 * kBWarps) == 0, "weight widening split");

struct Smem {
  uint32_t base;
  uint8_t* ptr;
  __device__ uint32_t bar(int i) const { return base + kOffBar + 8u * i; }
  __device__ uint32_t pk_full(int s) const { return bar(s); }
  __device__ uint32_t pk_empty(int s) const { return bar(kStages + s); }
  __device__ uint32_t op_empty(int s) const { return bar(2 * kStages + s); }  // MMA done with stage
  __device__ uint32_t ready(int s) const { return bar(3 * kStages + s); }     // this CTA widened
  __device__ uint32_t op_full(int s) const { return bar(4 * kStages + s); }   // leader: other CTA widened
  __device__ uint32_t acc_full(int b) const { return bar(5 * kStages + b); }
  __device__ uint32_t acc_empty(int b) const { return bar(5 * kStages + 2 + b); }
};

struct Problem {
  int M, N, K;
  int n_tiles, num_tiles, kblocks;
  int pair, num_pairs;
  uint32_t rank;
  __device__ void tile_origin(int t, int& m0, int& n0) const {
    m0 = (t / n_tiles) * BM;
    n0 = (t % n_tiles) * BN;
  }
};

__device__ __forceinline__ void producer_role(const Smem& sm, const Problem& pb,
                                              const CUtensorMap* tmA, const CUtensorMap* tmB,
                                              volatile int* abort_flag) {
  int s = 0;
  uint32_t ph = 0;
  for (int t = pb.pair; t < pb.num_tiles; t += pb.num_pairs) {
    int m0, n0;
    pb.tile_origin(t, m0, n0);
    for (int kb = 0; kb < pb.kblocks; ++kb) {
      if (!mbar_wait_bounded(sm.pk_empty(s), ph ^ 1u, abort_flag, kErrWaitProducer)) return;
      const uint32_t dst = sm.base + kOffPk + s * kPkStage;
      mbar_arrive_expect_tx(sm.pk_full(s), kPkStage);
      tma_load_2d(dst, tmA, kb * (BK / 2), m0 + static_cast<int>(pb.rank) * HM, sm.pk_full(s));
      tma_load_2d(dst + kPkA, tmB, kb * (BK / 2), n0 + static_cast<int>(pb.rank) * HN,
                  sm.pk_full(s));
      if (++s == kStages) { s = 0; ph ^= 1u; }
    }
  }
}

// One token row per thread: the row's 64 packed bytes of the stage (read from
// the 64-byte-swizzled tile: chunk j of row r at chunk j ^ ((r >> 1) & 3),
// conflict-free for 8 consecutive rows) widened to 32 columns of tensor memory.
__device__ __forceinline__ void widen_a_role(const Smem& sm, const Problem& pb, uint32_t tmem_base,
                                             int quad, int lane, volatile int* abort_flag) {
  const int r = 32 * quad + lane;
  const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(32 * quad) << 16);
  int s = 0;
  uint32_t ph = 0;
  for (int t = pb.pair; t < pb.num_tiles; t += pb.num_pairs) {
    for (int kb = 0; kb < pb.kblocks; ++kb) {
      // warp-uniform waits: the tensor-memory store below is .sync.aligned
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(sm.pk_full(s), ph, abort_flag,
                                                       kErrWaitUnpack)))
        return;
      const uint8_t* pk = sm.ptr + kOffPk + s * kPkStage + r * 64;
      uint4 w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        w[j] = *reinterpret_cast<const uint4*>(pk + ((j ^ ((r >> 1) & 3)) << 4));
      uint32_t c[32];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t v[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          c[8 * j + i] = (v[i] << 4) & 0xF0F0F0F0u;  // even elements
          c[8 * j + 4 + i] = v[i] & 0xF0F0F0F0u;     // odd elements
        }
      }
      // the stage's tensor-memory columns are free once the MMAs that read
      // them (k-block kb - kStages) have completed
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(sm.op_empty(s), ph ^ 1u, abort_flag,
                                                       kErrWaitUnpack)))
        return;
      tc_fence_after();
      tmem_st_32x32b_x32(lane_addr + static_cast<uint32_t>(kACol0 + kACols * s), c);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(sm.ready(s));
        mbar_arrive(sm.pk_empty(s));
      }
      if (++s == kStages) { s = 0; ph ^= 1u; }
    }
  }
}

// The weight tile: 96 rows x 4 packed chunks per stage, three chunks per
// thread, widened into the 128-byte-swizzled operand tile (16-byte chunk c of
// row r at chunk c ^ (r & 7)).
__device__ __forceinline__ void widen_b_role(const Smem& sm, const Problem& pb, int ut,
                                             volatile int* abort_flag) {
  const int lane = ut & 31;
  int s = 0;
  uint32_t ph = 0;
  for (int t = pb.pair; t < pb.num_tiles; t += pb.num_pairs) {
    for (int kb = 0; kb < pb.kblocks; ++kb) {
      if (!mbar_wait_bounded(sm.pk_full(s), ph, abort_flag, kErrWaitUnpack)) return;
      const uint8_t* pk = sm.ptr + kOffPk + s * kPkStage + kPkA;
      uint4 wv[kBChunksPerThread];
#pragma unroll
      for (int i = 0; i < kBChunksPerThread; ++i)
        wv[i] = *reinterpret_cast<const uint4*>(pk + (ut + i * 32 * kBWarps) * 16);
      if (!mbar_wait_bounded(sm.op_empty(s), ph ^ 1u, abort_flag, kErrWaitUnpack)) return;
      uint8_t* op = sm.ptr + kOffOp + s * kOpBytes;
#pragma unroll
      for (int i = 0; i < kBChunksPerThread; ++i) {
        const int c = ut + i * 32 * kBWarps;
        const int r = c >> 2;
        const int j = c & 3;
        const uint4 w = wv[i];
        const uint4 lo = make_uint4((w.x << 4) & 0xF0F0F0F0u, (w.y << 4) & 0xF0F0F0F0u,
                                    (w.z << 4) & 0xF0F0F0F0u, (w.w << 4) & 0xF0F0F0F0u);
        const uint4 hi = make_uint4(w.x & 0xF0F0F0F0u, w.y & 0xF0F0F0F0u, w.z & 0xF0F0F0F0u,
                                    w.w & 0xF0F0F0F0u);
        uint8_t* rowp = op + r * 128;
        *reinterpret_cast<uint4*>(rowp + (((2 * j) ^ (r & 7)) << 4)) = lo;
        *reinterpret_cast<uint4*>(rowp + (((2 * j + 1) ^ (r & 7)) << 4)) = hi;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(sm.ready(s));
        mbar_arrive(sm.pk_empty(s));
      }
      if (++s == kStages) { s = 0; ph ^= 1u; }
    }
  }
  // drain: every stage's last release has arrived before the CTA may exit
  if (lane == 0) {
    for (int i = 0; i < kStages; ++i) {
      if (!mbar_wait_bounded(sm.op_empty(s), ph ^ 1u, abort_flag, kErrWaitUnpack)) return;
      if (++s == kStages) { s = 0; ph ^= 1u; }
    }
  }
}

// Non-leader CTA: forwards "this CTA's stage is widened" (activation rows in
// its tensor memory, weight rows in its shared memory) to the leader's
// op_full barrier as a 16-byte bulk copy.
__device__ __forceinline__ void relay_role(const Smem& sm, const Problem& pb,
                                           volatile int* abort_flag) {
  int s = 0;
  uint32_t ph = 0;
  for (int t = pb.pair; t < pb.num_tiles; t += pb.num_pairs) {
    for (int kb = 0; kb < pb.kblocks; ++kb) {
      if (!mbar_wait_bounded(sm.ready(s), ph, abort_flag, kErrWaitUnpack)) return;
      tc_fence_after();
      const uint32_t slot = sm.base + kOffSignal + 16 * s;
      bulk_signal(map_to_rank(slot, 0), slot, map_to_rank(sm.op_full(s), 0));
      if (++s == kStages) { s = 0; ph ^= 1u; }
    }
  }
}

// Leader CTA only.
__device__ __forceinline__ void mma_role(const Smem& sm, const Problem& pb, uint32_t tmem_base,
                                         volatile int* abort_flag) {
  constexpr uint32_t idesc = idesc_i8(BM, BN);
  int s = 0;
  uint32_t ph = 0;
  int it = 0;
  for (int t = pb.pair; t < pb.num_tiles; t += pb.num_pairs, ++it) {
    const int buf = it & 1;
    const uint32_t aph = (it >> 1) & 1;
    if (!mbar_wait_cluster_bounded(sm.acc_empty(buf), aph ^ 1u, abort_flag, kErrWaitMma)) return;
    tc_fence_after();
    const uint32_t d = tmem_base + static_cast<uint32_t>(buf * kAccCols);
    for (int kb = 0; kb < pb.kblocks; ++kb) {
      mbar_arrive_expect_tx(sm.op_full(s), 16);  // the relay's signal
      if (!mbar_wait_bounded(sm.ready(s), ph, abort_flag, kErrWaitMma)) return;
      if (!mbar_wait_cluster_bounded(sm.op_full(s), ph, abort_flag, kErrWaitMma)) return;
      tc_fence_after();
      const uint32_t a0 = tmem_base + static_cast<uint32_t>(kACol0 + kACols * s);
      const uint32_t b0 = sm.base + kOffOp + s * kOpBytes;
#pragma unroll
      for (int kk = 0; kk < BK / 32; ++kk)
        mma_i8_pair_ts(d, a0 + 8 * kk, smem_desc_sw128(b0 + kk * 32), idesc, (kb | kk) != 0);
      mma_commit_both(sm.op_empty(s));
      if (++s == kStages) { s = 0; ph ^= 1u; }
    }
    mma_commit_both(sm.acc_full(buf));
  }
}

template <bool OUT_S32, bool ASYM>
__device__ __forceinline__ void epilogue_role(const Smem& sm, const Problem& pb,
                                              uint32_t tmem_base, int quad, int lane, int et,
                                              const float* __restrict__ sa,
                                              const float* __restrict__ sw,
                                              const uint16_t* __restrict__ bias,
                                              const int* __restrict__ rowsum,
                                              const int* __restrict__ offset, void* out,
                                              float* epi_sw, float* epi_b, int* epi_off,
                                              volatile int* abort_flag) {
  int it = 0;
  for (int t = pb.pair; t < pb.num_tiles; t += pb.num_pairs, ++it) {
    const int buf = it & 1;
    const uint32_t aph = (it >> 1) & 1;
    int m0, n0;
    pb.tile_origin(t, m0, n0);
    if (!OUT_S32 || ASYM) {
      gemm::epi_bar_sync();  // every epilogue warp is done with the previous tile's copy
      for (int i = et; i < BN; i += 32 * kEpiWarps) {
        const int n = n0 + i;
        const bool ok = n < pb.N;
        if (!OUT_S32) {
          epi_sw[i] = ok ? sw[n] : 0.f;
          epi_b[i] = (ok && bias) ? __uint_as_float(static_cast<uint32_t>(bias[n]) << 16) : 0.f;
        }
        if (ASYM) epi_off[i] = ok ? offset[n] : 0;
      }
      gemm::epi_bar_sync();
    }
    const int row = m0 + static_cast<int>(pb.rank) * HM + 32 * quad + lane;
    const bool row_ok = row < pb.M;
    const float s_a = (!OUT_S32 && row_ok) ? sa[row] : 0.f;
    const int rsum = (ASYM && row_ok) ? rowsum[row] : 0;
    if (!mbar_wait_bounded(sm.acc_full(buf), aph, abort_flag, kErrWaitEpilogue)) return;
    tc_fence_after();
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * quad) << 16) +
                           static_cast<uint32_t>(buf * kAccCols);
    const bool wide = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
    uint32_t ra[32], rb[32];
    tmem_ld_32x32b_x32(taddr, ra);
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < BN / 32; c += 2) {
      tmem_ld_32x32b_x32(taddr + 32 * (c + 1), rb);
      epilogue_chunk<kShift, OUT_S32, ASYM>(ra, row, row_ok, n0 + 32 * c, pb.N, s_a,
                                            epi_sw + 32 * c, epi_b + 32 * c, epi_off + 32 * c,
                                            rsum, out, wide);
      tmem_wait_ld();
      if (c + 2 < BN / 32) tmem_ld_32x32b_x32(taddr + 32 * (c + 2), ra);
      epilogue_chunk<kShift, OUT_S32, ASYM>(rb, row, row_ok, n0 + 32 * (c + 1), pb.N, s_a,
                                            epi_sw + 32 * (c + 1), epi_b + 32 * (c + 1),
                                            epi_off + 32 * (c + 1), rsum, out, wide);
      tmem_wait_ld();
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      if (pb.rank == 0)
        mbar_arrive(sm.acc_empty(buf));
      else
        mbar_arrive_cluster(map_to_rank(sm.acc_empty(buf), 0));
    }
  }
}

template <bool OUT_S32, bool ASYM>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    qgemm_ta_kernel(const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmB, const float* __restrict__ sa,
                    const float* __restrict__ sw, const uint16_t* __restrict__ bias, void* out,
                    int M, int N, int K, const int* gate, int gate_want,
                    const int* __restrict__ rowsum, const int* __restrict__ offset) {
  // a launch gated on a device-side width returns unless selected; both CTAs
  // of a pair read the same word, before any cluster or TMEM step
  if (gate != nullptr && *gate != gate_want) return;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  Smem sm;
  sm.ptr = smem_raw + pad;
  sm.base = raw + pad;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm.ptr + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm.ptr + kOffMisc + 4);

  Problem pb;
  pb.M = M;
  pb.N = N;
  pb.K = K;
  pb.n_tiles = (N + BN - 1) / BN;
  pb.num_tiles = ((M + BM - 1) / BM) * pb.n_tiles;
  pb.kblocks = K / BK;
  pb.rank = cluster_ctarank();
  pb.pair = blockIdx.x >> 1;
  pb.num_pairs = gridDim.x >> 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(sm.pk_full(s), 1);
      mbar_init(sm.pk_empty(s), kWidenWarps);
      mbar_init(sm.op_empty(s), 1);
      mbar_init(sm.ready(s), kWidenWarps);
      mbar_init(sm.op_full(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(sm.acc_full(b), 1);
      mbar_init(sm.acc_empty(b), 2 * kEpiWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) producer_role(sm, pb, &tmA, &tmB, abort_flag);
  } else if (warp == 1) {
    if (lane == 0 && pb.rank == 0) mma_role(sm, pb, tmem_base, abort_flag);
    if (lane == 0 && pb.rank != 0) relay_role(sm, pb, abort_flag);
  } else if (warp < 2 + kEpiWarps) {
    float* epi_sw = reinterpret_cast<float*>(sm.ptr + kOffEpi);
    epilogue_role<OUT_S32, ASYM>(sm, pb, tmem_base, warp & 3, lane, threadIdx.x - 64, sa, sw,
                                 bias, rowsum, offset, out, epi_sw, epi_sw + BN,
                                 reinterpret_cast<int*>(epi_sw + 2 * BN), abort_flag);
  } else if (warp < 2 + kEpiWarps + kAWarps) {
    widen_a_role(sm, pb, tmem_base, warp & 3, lane, abort_flag);
  } else {
    widen_b_role(sm, pb, threadIdx.x - 32 * (2 + kEpiWarps + kAWarps), abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its partner may still signal it
  if (*abort_flag) {
    // A wait gave up: give copies and MMAs already in flight time to land
    // before the tensor memory is released.
    const unsigned long long t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 2000000ull) __nanosleep(1000);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// Host side.  xp: packed activation codes [M][K/2]; wp: packed weight codes
// [N][K/2]; both 16-byte aligned rows (K % 128 == 0).
template <bool OUT_S32, bool ASYM = false>
inline qs_status launch_qgemm_ta(const void* xp, const float* sa, const void* wp,
                                 const float* sw, const void* bias, int64_t M, int64_t N,
                                 int64_t K, void* out, cudaStream_t stream,
                                 const int* gate = nullptr, int gate_want = 0,
                                 const int* rowsum = nullptr, const int* offset = nullptr) {
  CUtensorMap ta, tb;
  if (!make_tensor_map_2d_sw64(&ta, xp, static_cast<uint64_t>(K) / 2, static_cast<uint64_t>(M),
                               HM) ||
      !make_tensor_map_2d(&tb, wp, static_cast<uint64_t>(K) / 2, static_cast<uint64_t>(N),
                          BK / 2, HN, false))
    return QS_ERR_CUDA;
  auto kern = qgemm_ta_kernel<OUT_S32, ASYM>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
      cudaSuccess)
    return QS_ERR_CUDA;
  const int sms = sm_count();
  if (sms <= 0) return QS_ERR_CUDA;
  const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int64_t pairs = tiles < sms / 2 ? tiles : sms / 2;
  if (pairs < 1) return QS_ERR_CUDA;
  kern<<<static_cast<int>(2 * pairs), kThreads, kSmemBytes, stream>>>(
      ta, tb, sa, sw, static_cast<const uint16_t*>(bias), out, static_cast<int>(M),
      static_cast<int>(N), static_cast<int>(K), gate, gate_want, rowsum, offset);
  return cudaGetLastError() == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}

}  // namespace gemm_ta

namespace gemm {

// The GEMM form for the storage widths of the two operands: both packed
// 4-bit (the activation operand widened into tensor memory), both 8-bit, or
// mixed (the 4-bit one widened in shared memory).
template <bool OUT_S32>
inline qs_status dispatch_qgemm(int bits_x, int bits_w, const void* xp, const float* sa,
                                const void* wp,
                         const float* sw, const void* bias, int64_t M, int64_t N, int64_t K,
                         void* out, cudaStream_t stream) {
  // storage per code: 4-bit codes in nibbles, 6- and 8-bit codes in bytes
  const int sx = bits_x == 4 ? 4 : 8, sww = bits_w == 4 ? 4 : 8;
  if (sx == 4 && sww == 4)
    return gemm_ta::launch_qgemm_ta<OUT_S32>(xp, sa, wp, sw, bias, M, N, K, out, stream);
  if (sx == 8 && sww == 8)
    return launch_qgemm<8, 8, OUT_S32>(xp, sa, wp, sw, bias, M, N, K, out, stream);
  if (sx == 8 && sww == 4)
    return launch_qgemm<8, 4, OUT_S32>(xp, sa, wp, sw, bias, M, N, K, out, stream);
  return launch_qgemm<4, 8, OUT_S32>(xp, sa, wp, sw, bias, M, N, K, out, stream);
}

}  // namespace gemm
}  // namespace qs
