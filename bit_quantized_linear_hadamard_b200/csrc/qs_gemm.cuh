// Integer tensor-core GEMM with the dequantizing epilogue (tcgen05, sm_100a).
//
// The low-bit product of the rotated layer (DVD-Quant "Resumen técnico" §1 and
// §4: W4A4; §2.C: the 8-bit branch):
//   acc[m][n] = sum_k q_a[m][k] * q_w[n][k]                       (int32, exact)
//   out[m][n] = bf16(fl(fl(fl(s_a[m] * s_w[n]) * float(acc)) + bias[n]))
//
// Structure: a persistent kernel launched as clusters of two CTAs on the two
// SMs of a TPC.  Each pair walks output tiles of 256 x 512 (forms with a 4-bit
// operand) or 256 x 256 (the 8x8 form), n fastest, so the whole packed weight
// stays in L2 while activation tiles stream once (the 8-bit weight of the 8x8
// form is twice as large and is walked in bands of N-tiles instead, see
// kBandN).  CTA r of the pair holds rows [128r, 128r+128) of the x tile and,
// for each N-half h of the tile, rows [256h + 128r, 256h + 128r + 128) of the
// W tile; the leader (r = 0) issues per 32-deep K step one
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 32) per N-half, all reading
// the same x rows of both CTAs; each CTA's 128-row result accumulates in that
// CTA's tensor memory.  Per SM this halves the W operand traffic of a
// single-CTA tile at the same MMA work.  With two N-halves, one widening of a
// 4-bit x tile, one TMA load of x and one set of stage barriers serve twice
// the multiply-adds of a 256 x 256 tile.  (Measured: with the operand traffic
// of a 256 x 256 tile, issuing twice the MMAs per stage took 1.33x the time,
// at the tensor pipe's full rate; the smaller tile left it idle a third of its
// cycles.)
//
// Warp roles (both CTAs):
//   warp 0      TMA producer
//   warp 1      TMEM allocation; in the leader the single-thread MMA issuer;
//               in the other CTA (4-bit only) the relay that tells the leader
//               that this CTA's operand tiles are ready
//   warps 2-9   epilogue (2-5 in the 8x8 form): tcgen05.ld of this CTA's
//               accumulator rows, scale, bias, bf16 store; warps 2-5 the first
//               N-half, 6-9 the second
//   warps 10-13 (4-bit only) widen packed nibbles into the 8-bit operand tiles
// With 256 x 512 tiles the 128 x 512 int32 accumulator fills the 512 TMEM
// columns, so the MMA of the next tile waits for the epilogue to drain it (the
// operand ring keeps filling meanwhile); the 8x8 form's 256-column
// accumulators are two, so its epilogue runs under the next tile's main loop.
//
// Synchronisation across the pair: 8-bit operand stages are "full" on the
// leader's barrier when the TMA loads of both CTAs have landed.  4-bit operand
// stages are "unpacked" on a local barrier of each CTA; the other CTA's relay
// thread forwards its local completion to the leader's "full" barrier as a
// 16-byte shared-to-shared bulk copy whose transaction bytes complete that
// barrier.  (A software cluster-scope release per stage instead stalls the
// arriving thread for a memory-barrier round trip every stage, which measured
// as the limit of the whole main loop.)  The leader's MMA
// completion is committed to the "empty" barrier of both CTAs with one
// multicast commit per stage (two separate commits cost the tensor pipe 3-5 %
// of the main loop); accumulator readiness likewise goes to both CTAs; the
// epilogue warps of both CTAs arrive on the leader's "accumulator free"
// barrier.
//
// 4-bit operands: tcgen05 has no 4-bit integer kind, so each packed 16-byte
// chunk (32 nibbles = 32 consecutive K elements) is widened in shared memory to
// 32 bytes: the low nibbles (even elements) as one 16-byte chunk and the high
// nibbles (odd elements) as the next, each nibble placed in the HIGH half of
// its byte.  That byte, read as int8, is 16*q exactly, so the tensor core
// accumulates 256*acc; the epilogue shifts it back (exact).  Both operands get
// the same K permutation, so every dot product is unchanged.  The widening is
// one shift and one mask per 4 output bytes.  When only one operand is 4-bit
// the other is in natural K order, so the widened bytes are interleaved back
// into natural order (two byte permutes more per 8 output bytes).
// |16 q| <= 112 keeps 256*acc inside int32 for K <= 65536.
//
// 8-bit operands go from global memory to the 128-byte-swizzled operand tiles
// directly by TMA.  (6-bit codes are stored as int8 and take this path.)
//
// Mixed widths (W4A8 of QuantSparse, W4A6 of DVD-Quant, both "Resumen
// técnico" §4; 8-bit storage for x, 4-bit for W): the 8-bit operand is loaded
// by TMA straight into its half of the operand stage and the 4-bit one is
// widened into the other half.  The leader's producer arms its "full" barrier
// with the direct bytes of both CTAs plus the relay's 16 bytes; the MMA
// additionally waits for its own CTA's widening.  Only the widened operand carries the factor 16, so the epilogue
// shifts by 4 bits per 4-bit operand.
#pragma once

#include <cuda_bf16.h>

#include "qs.h"
#include "qs_host.cuh"
#include "qs_ptx.cuh"

namespace qs {
namespace gemm {

constexpr int BM = 256;  // tile rows (tokens), 128 per CTA
constexpr int NH = 256;  // columns of one MMA (an N-half of a tile)
constexpr int HM = 128;  // x rows per CTA
constexpr int HN = 128;  // W rows per CTA and N-half
constexpr int BK = 128;  // K elements per pipeline stage (= 128 bytes of 8-bit operand)
constexpr int kTmemCols = 512;  // all of tensor memory: int32 accumulator columns

// SA, SB: storage bits of the x and W codes (4 = two per byte, 8 = one byte).
template <int SA, int SB>
struct Cfg {
  static_assert((SA == 4 || SA == 8) && (SB == 4 || SB == 8), "storage is 4 or 8 bits");
  static constexpr bool kPackedA = SA == 4;
  static constexpr bool kPackedB = SB == 4;
  static constexpr bool kPacked = kPackedA || kPackedB;   // some operand is widened
  static constexpr bool kAllPacked = kPackedA && kPackedB;
  static constexpr bool kDirect = !kAllPacked;            // some operand goes by TMA directly
  // N-halves per tile: 2 (tiles of 256 x 512) when an operand is widened;
  // the 8x8 form keeps tiles of 256 x 256 with two accumulators (see kBandN)
  static constexpr int kHalves = kPacked ? 2 : 1;
  static constexpr int kBN = kHalves * NH;               // tile columns
  static constexpr int kAccBufs = kTmemCols / kBN;       // accumulators in tensor memory
  static constexpr int kPkBytesA = kPackedA ? HM * BK / 2 : 0;  // packed tile of x (this CTA)
  static constexpr int kPkBytesB = kPackedB ? kHalves * HN * BK / 2 : 0;  // packed W tiles
  static constexpr int kOpBytesA = HM * BK;            // 8-bit operand tile of x
  static constexpr int kOpBytesB = kHalves * HN * BK;  // 8-bit operand tiles of W
  static constexpr int kPkStage = kPkBytesA + kPkBytesB;
  static constexpr int kOpStage = kOpBytesA + kOpBytesB;
  // bytes the TMA writes straight into one operand stage of this CTA
  static constexpr int kDirectBytes = (kPackedA ? 0 : kOpBytesA) + (kPackedB ? 0 : kOpBytesB);
  // as many stages as fit in shared memory
  static constexpr int kOpStages = kPacked ? 3 : 6;
  static constexpr int kPkStages = kPacked ? kOpStages : 0;  // one ring index drives both
  static constexpr int kEpiWarps = 4 * kHalves;  // per TMEM lane quarter, one per N-half
  static constexpr int kUnpackWarps = kPacked ? 4 : 0;
  // operand-tile row that packed row 0 widens into (W rows follow the 128 x rows)
  static constexpr int kUnpackRow0 = kPackedA ? 0 : HM;
  // the tensor core sees 16 q for every widened operand
  static constexpr int kAccShift = 4 * (static_cast<int>(kPackedA) + static_cast<int>(kPackedB));
  static constexpr int kThreads = 32 * (2 + kEpiWarps + kUnpackWarps);
  static constexpr int kOffOp = 0;
  static constexpr int kOffPk = kOffOp + kOpStages * kOpStage;
  static constexpr int kOffBar = kOffPk + kPkStages * kPkStage;
  static constexpr int kNumBars = 2 * kPkStages + 3 * kOpStages + 4;
  // s_w, bias and (asymmetric weights) channel offsets of a tile
  static constexpr int kOffEpi = (kOffBar + 8 * kNumBars + 15) / 16 * 16;
  static constexpr int kOffMisc = kOffEpi + 3 * kBN * 4;  // TMEM address, abort flag
  static constexpr int kOffSignal = kOffMisc + 16;        // 16 bytes per operand stage
  static constexpr int kSmemBytes = kOffSignal + 16 * kOpStages + 1024;  // + alignment slack
  static constexpr int kUnpackThreads = kPacked ? 32 * kUnpackWarps : 1;
  static constexpr int kChunksPerThread = kPacked ? (kPkStage / 16) / kUnpackThreads : 0;
  static_assert((kPkStage / 16) % kUnpackThreads == 0, "unpack split");
  // arrivals completing one "operand full" phase on the leader: its MMA
  // thread arming the relay's 16 bytes (both operands 4-bit) or its producer
  // arming both CTAs' direct TMA bytes (+ the relay's 16 bytes when mixed)
  static constexpr int kOpFullCount = 1;
  static constexpr int kOpFullTx = 2 * kDirectBytes + (kPacked ? 16 : 0);
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
  static constexpr int kAccEmptyCount = 2 * kEpiWarps;
  static constexpr int kEpiThreads = 32 * kEpiWarps;
};

struct Smem {
  uint32_t base;  // shared-window address of the 1024-aligned layout (this CTA)
  uint8_t* ptr;
  int P, U;
  uint32_t off_bar;
  __device__ uint32_t bar(int i) const { return base + off_bar + 8u * i; }
  __device__ uint32_t pk_full(int s) const { return bar(s); }
  __device__ uint32_t pk_empty(int s) const { return bar(P + s); }
  __device__ uint32_t op_full(int s) const { return bar(2 * P + s); }
  __device__ uint32_t op_empty(int s) const { return bar(2 * P + U + s); }
  __device__ uint32_t acc_full(int b) const { return bar(2 * P + 2 * U + b); }
  __device__ uint32_t acc_empty(int b) const { return bar(2 * P + 2 * U + 2 + b); }
  __device__ uint32_t unpacked(int s) const { return bar(2 * P + 2 * U + 4 + s); }
};

// Tile order of the 8-bit x 8-bit instantiation: bands of kBandN N-tiles,
// M advancing inside a band, so that the band's slice of the 8-bit weight
// (18 x 256 rows, 23.6 MB at K = 5120) stays in L2 while the activation tiles
// stream.  In n-fastest order the whole 70.8 MB weight of the Wan FFN was read
// from DRAM about 19 times per launch; banded, the launch measured 5-10 %
// faster.  The other instantiations, whose packed 4-bit weight fits in L2,
// keep the n-fastest order.  (The 8x8 form keeps tiles of 256 x 256: with
// 256 x 512 tiles it measured 1.478 against 1.395 ms at the Wan FFN shape,
// where it runs at the board's power limit.)
constexpr int kBandN = 18;

struct Problem {
  int M, N, K;
  int bn;               // tile columns
  int n_tiles, num_tiles, kblocks;
  int band;             // N-tiles per band, 0: n-fastest order
  int pair, num_pairs;  // this pair's index and the number of pairs
  uint32_t rank;        // 0 = leader
  __device__ void tile_origin(int t, int& m0, int& n0) const {
    if (band > 0) {
      const int m_tiles = num_tiles / n_tiles;
      const int per_band = band * m_tiles;
      const int g = t / per_band, r = t - g * per_band;
      const int gn = min(band, n_tiles - g * band);  // the last band may be narrower
      m0 = (r / gn) * BM;
      n0 = (g * band + r % gn) * bn;
    } else {
      m0 = (t / n_tiles) * BM;
      n0 = (t % n_tiles) * bn;
    }
  }
};

template <int SA, int SB>
__device__ __forceinline__ void producer_role(const Smem& sm, const Problem& pb,
                                              const CUtensorMap* tmA, const CUtensorMap* tmB,
                                              volatile int* abort_flag) {
  using C = Cfg<SA, SB>;
  int s = 0;
  uint32_t ph = 0;
  const int roff = static_cast<int>(pb.rank) * HM;
  for (int t = pb.pair; t < pb.num_tiles; t += pb.num_pairs) {
    int m0, n0;
    pb.tile_origin(t, m0, n0);
    for (int kb = 0; kb < pb.kblocks; ++kb) {
      if (C::kPacked) {
        // packed tiles stay in this CTA: ordinary loads on a local barrier
        if (!mbar_wait_bounded(sm.pk_empty(s), ph ^ 1u, abort_flag, kErrWaitProducer)) return;
        const uint32_t dst = sm.base + C::kOffPk + s * C::kPkStage;
        mbar_arrive_expect_tx(sm.pk_full(s), C::kPkStage);
        if (C::kPackedA) tma_load_2d(dst, tmA, kb * (BK / 2), m0 + roff, sm.pk_full(s));
        if (C::kPackedB)
#pragma unroll
          for (int h = 0; h < C::kHalves; ++h)
            tma_load_2d(dst + C::kPkBytesA + h * (HN * BK / 2), tmB, kb * (BK / 2),
                        n0 + h * NH + roff, sm.pk_full(s));
      }
      if (C::kDirect) {
        // direct operand tiles of both CTAs complete on the leader's barrier
        if (!mbar_wait_bounded(sm.op_empty(s), ph ^ 1u, abort_flag, kErrWaitProducer)) return;
        const uint32_t dst = sm.base + C::kOffOp + s * C::kOpStage;
        const uint32_t full_leader = map_to_rank(sm.op_full(s), 0);
        if (pb.rank == 0) mbar_arrive_expect_tx(sm.op_full(s), C::kOpFullTx);
        if (!C::kPackedA) tma_load_2d_pair(dst, tmA, kb * BK, m0 + roff, full_leader);
        if (!C::kPackedB)
#pragma unroll
          for (int h = 0; h < C::kHalves; ++h)
            tma_load_2d_pair(dst + C::kOpBytesA + h * (HN * BK), tmB, kb * BK,
                             n0 + h * NH + roff, full_leader);
      }
      if (++s == C::kOpStages) { s = 0; ph ^= 1u; }
    }
  }
  if (!C::kPacked) {
    // drain: every stage's last release has arrived before the CTA may exit
    for (int i = 0; i < C::kOpStages; ++i) {
      if (!mbar_wait_bounded(sm.op_empty(s), ph ^ 1u, abort_flag, kErrWaitProducer)) return;
      if (++s == C::kOpStages) { s = 0; ph ^= 1u; }
    }
  }
}

// Widens packed 4-bit tiles into 8-bit operand tiles (see the file comment).
// Packed stage: the 4-bit tiles among [x tile 128 rows x 64 B][W tiles of the
// two N-halves, 2 x 128 rows x 64 B], plain rows.  Operand stage: [x tile 128
// rows x 128 B][W tiles 2 x 128 rows x 128 B], rows of 128 B with 16-byte
// chunk c stored at chunk c ^ (row & 7) (128-byte swizzle).
template <int SA, int SB>
__device__ __forceinline__ void unpack_role(const Smem& sm, const Problem& pb, int ut,
                                            volatile int* abort_flag) {
  using C = Cfg<SA, SB>;
  const int lane = ut & 31;
  int sp = 0, su = 0;
  uint32_t php = 0, phu = 0;
  for (int t = pb.pair; t < pb.num_tiles; t += pb.num_pairs) {
    for (int kb = 0; kb < pb.kblocks; ++kb) {
      if (!mbar_wait_bounded(sm.pk_full(sp), php, abort_flag, kErrWaitUnpack)) return;
      if (!mbar_wait_bounded(sm.op_empty(su), phu ^ 1u, abort_flag, kErrWaitUnpack)) return;
      const uint8_t* pk = sm.ptr + C::kOffPk + sp * C::kPkStage;
      uint8_t* op = sm.ptr + C::kOffOp + su * C::kOpStage;
      // all loads first: they are independent of the stores that follow
      uint4 wv[C::kChunksPerThread > 0 ? C::kChunksPerThread : 1];
#pragma unroll
      for (int i = 0; i < C::kChunksPerThread; ++i)
        wv[i] = *reinterpret_cast<const uint4*>(pk + (ut + i * C::kUnpackThreads) * 16);
#pragma unroll
      for (int i = 0; i < C::kChunksPerThread; ++i) {
        const int c = ut + i * C::kUnpackThreads;
        const uint4 w = wv[i];
        const int r = C::kUnpackRow0 + (c >> 2);  // operand row (x rows 0..127, then W rows)
        const int j = c & 3;   // packed 16-byte chunk within the row's 64 bytes
        uint4 lo, hi;
        lo.x = (w.x << 4) & 0xF0F0F0F0u;
        lo.y = (w.y << 4) & 0xF0F0F0F0u;
        lo.z = (w.z << 4) & 0xF0F0F0F0u;
        lo.w = (w.w << 4) & 0xF0F0F0F0u;
        hi.x = w.x & 0xF0F0F0F0u;
        hi.y = w.y & 0xF0F0F0F0u;
        hi.z = w.z & 0xF0F0F0F0u;
        hi.w = w.w & 0xF0F0F0F0u;
        if (!C::kAllPacked) {
          // the other operand is in natural K order: interleave the low-nibble
          // (even) and high-nibble (odd) bytes back to elements 0..15, 16..31
          const uint4 l = lo, h = hi;
          lo = make_uint4(__byte_perm(l.x, h.x, 0x5140), __byte_perm(l.x, h.x, 0x7362),
                          __byte_perm(l.y, h.y, 0x5140), __byte_perm(l.y, h.y, 0x7362));
          hi = make_uint4(__byte_perm(l.z, h.z, 0x5140), __byte_perm(l.z, h.z, 0x7362),
                          __byte_perm(l.w, h.w, 0x5140), __byte_perm(l.w, h.w, 0x7362));
        }
        uint8_t* rowp = op + r * 128;
        *reinterpret_cast<uint4*>(rowp + (((2 * j) ^ (r & 7)) << 4)) = lo;
        *reinterpret_cast<uint4*>(rowp + (((2 * j + 1) ^ (r & 7)) << 4)) = hi;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(sm.unpacked(su));
        mbar_arrive(sm.pk_empty(sp));
      }
      if (++sp == C::kPkStages) { sp = 0; php ^= 1u; }
      if (++su == C::kOpStages) { su = 0; phu ^= 1u; }
    }
  }
  // drain: every operand stage's last release has arrived before the CTA may exit
  if (lane == 0) {
    for (int i = 0; i < C::kOpStages; ++i) {
      if (!mbar_wait_bounded(sm.op_empty(su), phu ^ 1u, abort_flag, kErrWaitUnpack)) return;
      if (++su == C::kOpStages) { su = 0; phu ^= 1u; }
    }
  }
}

// A 4-bit operand, non-leader CTA only: forwards "this CTA's operand stage is unpacked"
// to the leader's "full" barrier with one 16-byte signalling bulk copy per
// stage (the leader's MMA thread arms that barrier with the 16 bytes).
template <int SA, int SB>
__device__ __forceinline__ void relay_role(const Smem& sm, const Problem& pb,
                                           volatile int* abort_flag) {
  using C = Cfg<SA, SB>;
  int s = 0;
  uint32_t ph = 0;
  for (int t = pb.pair; t < pb.num_tiles; t += pb.num_pairs) {
    for (int kb = 0; kb < pb.kblocks; ++kb) {
      if (!mbar_wait_bounded(sm.unpacked(s), ph, abort_flag, kErrWaitUnpack)) return;
      const uint32_t slot = sm.base + C::kOffSignal + 16 * s;
      bulk_signal(map_to_rank(slot, 0), slot, map_to_rank(sm.op_full(s), 0));
      if (++s == C::kOpStages) { s = 0; ph ^= 1u; }
    }
  }
}

// Leader CTA only.
template <int SA, int SB>
__device__ __forceinline__ void mma_role(const Smem& sm, const Problem& pb, uint32_t tmem_base,
                                         volatile int* abort_flag) {
  using C = Cfg<SA, SB>;
  constexpr uint32_t idesc = idesc_i8(BM, NH);
  int s = 0;
  uint32_t ph = 0;
  int it = 0;
  for (int t = pb.pair; t < pb.num_tiles; t += pb.num_pairs, ++it) {
    const int buf = it % C::kAccBufs;
    const uint32_t aph = (it / C::kAccBufs) & 1;
    if (!mbar_wait_cluster_bounded(sm.acc_empty(buf), aph ^ 1u, abort_flag, kErrWaitMma)) return;
    tc_fence_after();
    const uint32_t d = tmem_base + static_cast<uint32_t>(buf * C::kBN);
    for (int kb = 0; kb < pb.kblocks; ++kb) {
      if (C::kAllPacked) mbar_arrive_expect_tx(sm.op_full(s), 16);  // the relay's signal
      if (C::kPacked && !mbar_wait_bounded(sm.unpacked(s), ph, abort_flag, kErrWaitMma)) return;
      if (!mbar_wait_cluster_bounded(sm.op_full(s), ph, abort_flag, kErrWaitMma)) return;
      tc_fence_after();
      const uint32_t a0 = sm.base + C::kOffOp + s * C::kOpStage;
      const uint32_t b0 = a0 + C::kOpBytesA;
      // both N-halves read the same x tile
#pragma unroll
      for (int kk = 0; kk < BK / 32; ++kk) {
        const uint64_t adesc = smem_desc_sw128(a0 + kk * 32);
#pragma unroll
        for (int h = 0; h < C::kHalves; ++h)
          mma_i8_pair(d + h * NH, adesc, smem_desc_sw128(b0 + h * (HN * BK) + kk * 32), idesc,
                      (kb | kk) != 0);
      }
      mma_commit_both(sm.op_empty(s));
      if (++s == C::kOpStages) { s = 0; ph ^= 1u; }
    }
    mma_commit_both(sm.acc_full(buf));
  }
}

// named barrier 1 over the epilogue warps only
template <int THREADS>
__device__ __forceinline__ void epi_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(THREADS) : "memory");
}

__device__ __forceinline__ void st_stream_v4(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

// 32-byte streaming store (one whole sector per lane); p 32-byte aligned.
__device__ __forceinline__ void st_stream_v8(void* p, const uint32_t (&v)[8]) {
  asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

// Converts one 32-column chunk of accumulators (one row per thread) and stores it.
// ASYM (weights on an asymmetric grid, signed codes s = q - 2^(b-1)): the
// exact accumulator is sum q_a s + o[n] * sum_k q_a[m,k].
// wide: `out` is 32-byte aligned, so 16 bf16 outputs go out as one 32-byte
// store (rows are 2N bytes apart with N % 16 == 0, chunks start at multiples
// of 32 columns); otherwise as two 16-byte stores.
template <int SHIFT, bool OUT_S32, bool ASYM>
__device__ __forceinline__ void epilogue_chunk(const uint32_t (&r)[32], int row, bool row_ok,
                                               int n, int N, float s_a, const float* epi_sw,
                                               const float* epi_b, const int* epi_off,
                                               int rsum, void* out, bool wide) {
  if (n >= N || !row_ok) return;
  int32_t acc[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    acc[i] = static_cast<int32_t>(r[i]) >> SHIFT;
    if (ASYM) acc[i] += epi_off[i] * rsum;
  }
  if (OUT_S32) {
    int32_t* dst = static_cast<int32_t*>(out) + static_cast<int64_t>(row) * N + n;
#pragma unroll
    for (int v = 0; v < 8; ++v)
      if (n + 4 * v + 4 <= N)
        st_stream_v4(dst + 4 * v, make_uint4(acc[4 * v], acc[4 * v + 1], acc[4 * v + 2],
                                             acc[4 * v + 3]));
  } else {
    uint16_t* dst = static_cast<uint16_t*>(out) + static_cast<int64_t>(row) * N + n;
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      if (n + 16 * v + 16 > N) break;  // N % 16 == 0: only whole 16-column groups exist
      uint32_t packed[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 w4 = *reinterpret_cast<const float4*>(epi_sw + 16 * v + 4 * q);
        const float4 b4 = *reinterpret_cast<const float4*>(epi_b + 16 * v + 4 * q);
        const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
        const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
          float y[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float sab = __fmul_rn(s_a, wv[e + h]);
            const float p = __fmul_rn(sab, __int2float_rn(acc[16 * v + 4 * q + e + h]));
            y[h] = __fadd_rn(p, bv[e + h]);
          }
          const __nv_bfloat162 y2 = __floats2bfloat162_rn(y[0], y[1]);
          packed[2 * q + (e >> 1)] = *reinterpret_cast<const uint32_t*>(&y2);
        }
      }
      if (wide) {
        st_stream_v8(dst + 16 * v, packed);
      } else {
        st_stream_v4(dst + 16 * v, make_uint4(packed[0], packed[1], packed[2], packed[3]));
        st_stream_v4(dst + 16 * v + 8, make_uint4(packed[4], packed[5], packed[6], packed[7]));
      }
    }
  }
}

// Epilogue warp (quad, ch): TMEM lanes 32 quad .. 32 quad + 31 (its rows)
// and the accumulator columns of N-half ch; et = 0 .. 32 EPI_WARPS - 1.
template <int SHIFT, bool OUT_S32, bool ASYM, int EPI_WARPS, int ACC_BUFS>
__device__ __forceinline__ void epilogue_role(const Smem& sm, const Problem& pb,
                                              uint32_t tmem_base, int quad, int ch, int lane,
                                              int et,
                                              const float* __restrict__ sa,
                                              const float* __restrict__ sw,
                                              const uint16_t* __restrict__ bias,
                                              const int* __restrict__ rowsum,
                                              const int* __restrict__ offset, void* out,
                                              float* epi_sw, float* epi_b, int* epi_off,
                                              volatile int* abort_flag) {
  int it = 0;
  for (int t = pb.pair; t < pb.num_tiles; t += pb.num_pairs, ++it) {
    const int buf = it % ACC_BUFS;
    const uint32_t aph = (it / ACC_BUFS) & 1;
    int m0, n0;
    pb.tile_origin(t, m0, n0);
    if (!OUT_S32 || ASYM) {
      // Stage the tile's channel scales, bias and offsets while its main loop runs.
      epi_bar_sync<32 * EPI_WARPS>();  // every epilogue warp is done with the previous copy
      for (int i = et; i < pb.bn; i += 32 * EPI_WARPS) {
        const int n = n0 + i;
        const bool ok = n < pb.N;
        if (!OUT_S32) {
          epi_sw[i] = ok ? sw[n] : 0.f;
          epi_b[i] = (ok && bias) ? __uint_as_float(static_cast<uint32_t>(bias[n]) << 16) : 0.f;
        }
        if (ASYM) epi_off[i] = ok ? offset[n] : 0;
      }
      epi_bar_sync<32 * EPI_WARPS>();
    }
    const int row = m0 + static_cast<int>(pb.rank) * HM + 32 * quad + lane;
    const bool row_ok = row < pb.M;
    const float s_a = (!OUT_S32 && row_ok) ? sa[row] : 0.f;
    const int rsum = (ASYM && row_ok) ? rowsum[row] : 0;
    if (!mbar_wait_bounded(sm.acc_full(buf), aph, abort_flag, kErrWaitEpilogue)) return;
    tc_fence_after();
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * quad) << 16) +
                           static_cast<uint32_t>(buf * pb.bn + ch * NH);
    // this warp's columns: n0 + ch NH .. + NH - 1
    n0 += ch * NH;
    const float* e_sw = epi_sw + ch * NH;
    const float* e_b = epi_b + ch * NH;
    const int* e_off = epi_off + ch * NH;
    // Two register sets: the TMEM load of chunk c+1 is in flight while chunk c
    // is converted and stored.
    const bool wide = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
    uint32_t ra[32], rb[32];
    tmem_ld_32x32b_x32(taddr, ra);
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < NH / 32; c += 2) {
      tmem_ld_32x32b_x32(taddr + 32 * (c + 1), rb);
      epilogue_chunk<SHIFT, OUT_S32, ASYM>(ra, row, row_ok, n0 + 32 * c, pb.N, s_a,
                                          e_sw + 32 * c, e_b + 32 * c, e_off + 32 * c,
                                          rsum, out, wide);
      tmem_wait_ld();
      if (c + 2 < NH / 32) tmem_ld_32x32b_x32(taddr + 32 * (c + 2), ra);
      epilogue_chunk<SHIFT, OUT_S32, ASYM>(rb, row, row_ok, n0 + 32 * (c + 1), pb.N, s_a,
                                          e_sw + 32 * (c + 1), e_b + 32 * (c + 1),
                                          e_off + 32 * (c + 1), rsum, out, wide);
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

template <int SA, int SB, bool OUT_S32, bool ASYM>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg<SA, SB>::kThreads, 1)
    qgemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const float* __restrict__ sa, const float* __restrict__ sw,
                 const uint16_t* __restrict__ bias, void* out, int M, int N, int K,
                 const int* gate, int gate_want, const int* __restrict__ rowsum,
                 const int* __restrict__ offset) {
  using C = Cfg<SA, SB>;
  // a launch gated on a device-side width (δ-GBS) returns unless selected;
  // both CTAs of a pair read the same word, before any cluster or TMEM step
  if (gate != nullptr && *gate != gate_want) return;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The padding is identical in both CTAs (same kernel, same static layout),
  // so every shared object has the same offset in the two CTAs of a pair.
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  Smem sm;
  sm.ptr = smem_raw + pad;
  sm.base = raw + pad;
  sm.P = C::kPkStages;
  sm.U = C::kOpStages;
  sm.off_bar = C::kOffBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm.ptr + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm.ptr + C::kOffMisc + 4);

  Problem pb;
  pb.M = M;
  pb.N = N;
  pb.K = K;
  pb.bn = C::kBN;
  pb.n_tiles = (N + C::kBN - 1) / C::kBN;
  pb.num_tiles = ((M + BM - 1) / BM) * pb.n_tiles;
  pb.kblocks = K / BK;
  pb.band = (SA == 8 && SB == 8) ? kBandN : 0;
  pb.rank = cluster_ctarank();
  pb.pair = blockIdx.x >> 1;
  pb.num_pairs = gridDim.x >> 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kPkStages; ++s) {
      mbar_init(sm.pk_full(s), 1);
      mbar_init(sm.pk_empty(s), C::kUnpackWarps);
    }
    for (int s = 0; s < C::kOpStages; ++s) {
      mbar_init(sm.op_full(s), C::kOpFullCount);
      mbar_init(sm.op_empty(s), 1);
    }
    for (int b = 0; b < C::kAccBufs; ++b) {
      mbar_init(sm.acc_full(b), 1);
      mbar_init(sm.acc_empty(b), C::kAccEmptyCount);
    }
    if (C::kPacked)
      for (int s = 0; s < C::kOpStages; ++s) mbar_init(sm.unpacked(s), C::kUnpackWarps);
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
    if (lane == 0) producer_role<SA, SB>(sm, pb, &tmA, &tmB, abort_flag);
  } else if (warp == 1) {
    if (lane == 0 && pb.rank == 0) mma_role<SA, SB>(sm, pb, tmem_base, abort_flag);
    if (lane == 0 && pb.rank != 0 && C::kPacked) relay_role<SA, SB>(sm, pb, abort_flag);
  } else if (warp < 2 + C::kEpiWarps) {
    float* epi_sw = reinterpret_cast<float*>(sm.ptr + C::kOffEpi);
    epilogue_role<C::kAccShift, OUT_S32, ASYM, C::kEpiWarps, C::kAccBufs>(
        sm, pb, tmem_base, warp & 3, (warp - 2) >> 2, lane, threadIdx.x - 64, sa, sw, bias,
        rowsum, offset, out, epi_sw, epi_sw + C::kBN,
        reinterpret_cast<int*>(epi_sw + 2 * C::kBN), abort_flag);
  } else {
    if (C::kPacked) unpack_role<SA, SB>(sm, pb, threadIdx.x - 32 * (2 + C::kEpiWarps), abort_flag);
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

// ---------------------------------------------------------------- launches
// (host side, here with the kernel so that both are one unit of the source)

// SA, SB: storage bits (4 or 8) of the x and W codes.  ASYM: weights on an
// asymmetric grid (per-token code sums `rowsum`, per-channel `offset`).
template <int SA, int SB, bool OUT_S32, bool ASYM = false>
inline qs_status launch_qgemm(const void* xp, const float* sa, const void* wp, const float* sw,
                       const void* bias, int64_t M, int64_t N, int64_t K, void* out,
                       cudaStream_t stream, const int* gate = nullptr, int gate_want = 0,
                       const int* rowsum = nullptr, const int* offset = nullptr) {
  using C = Cfg<SA, SB>;
  CUtensorMap ta, tb;
  // each CTA of a pair loads 128 rows of x and 128 rows of W per stage; 8-bit
  // tiles land 128-byte swizzled in the operand stage, 4-bit ones as plain rows
  if (!make_tensor_map_2d(&ta, xp, static_cast<uint64_t>(K) * SA / 8, static_cast<uint64_t>(M),
                              BK * SA / 8, HM, SA == 8) ||
      !make_tensor_map_2d(&tb, wp, static_cast<uint64_t>(K) * SB / 8, static_cast<uint64_t>(N),
                              BK * SB / 8, HN, SB == 8))
    return QS_ERR_CUDA;
  auto kern = qgemm_kernel<SA, SB, OUT_S32, ASYM>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
      cudaSuccess)
    return QS_ERR_CUDA;
  const int sms = sm_count();
  if (sms <= 0) return QS_ERR_CUDA;
  // persistent clusters of two CTAs, at most one CTA per SM
  const int64_t tiles = ((M + BM - 1) / BM) *
                        ((N + C::kBN - 1) / C::kBN);
  const int64_t pairs = tiles < sms / 2 ? tiles : sms / 2;
  if (pairs < 1) return QS_ERR_CUDA;
  const int grid = static_cast<int>(2 * pairs);
  kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(
      ta, tb, sa, sw, static_cast<const uint16_t*>(bias), out, static_cast<int>(M),
      static_cast<int>(N), static_cast<int>(K), gate, gate_want, rowsum, offset);
  return cudaGetLastError() == cudaSuccess ? QS_OK : QS_ERR_CUDA;
}

template <bool OUT_S32>
inline qs_status dispatch_qgemm(int bits_x, int bits_w, const void* xp, const float* sa,
                                const void* wp,
                         const float* sw, const void* bias, int64_t M, int64_t N, int64_t K,
                         void* out, cudaStream_t stream) {
  // storage per code: 4-bit codes in nibbles, 6- and 8-bit codes in bytes
  const int sx = bits_x == 4 ? 4 : 8, sww = bits_w == 4 ? 4 : 8;
  if (sx == 4 && sww == 4)
    return launch_qgemm<4, 4, OUT_S32>(xp, sa, wp, sw, bias, M, N, K, out, stream);
  if (sx == 8 && sww == 8)
    return launch_qgemm<8, 8, OUT_S32>(xp, sa, wp, sw, bias, M, N, K, out, stream);
  if (sx == 8 && sww == 4)
    return launch_qgemm<8, 4, OUT_S32>(xp, sa, wp, sw, bias, M, N, K, out, stream);
  return launch_qgemm<4, 8, OUT_S32>(xp, sa, wp, sw, bias, M, N, K, out, stream);
}

}  // namespace gemm
}  // namespace qs
