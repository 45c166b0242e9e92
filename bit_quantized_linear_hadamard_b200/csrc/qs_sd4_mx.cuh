// SD4 layer GEMM on the block-scaled fp8 tensor-core path.
//
// An SD4 value is (-1)^s L/8 2^e with L <= 15 and one power-of-two scale per
// 32 consecutive elements of a row: L/8 is an e4m3 number exactly (at most 4
// significant bits, exponent -3..0) and 2^e is a UE8M0 scale (e + 127,
// e in [-126, 127]).  That is the operand format of
// tcgen05.mma.kind::mxf8f6f4.block_scale with one scale per 32 elements along
// K, so the products x_hat * w_hat come out of the tensor cores exactly and
// are summed with binary32 accumulation, at the fp8 rate and with one byte
// per operand element in shared memory (the bf16 form needs two).
//
// Persistent, one CTA per SM, tiles of 128 x 192 (two 192-column binary32
// accumulators and the 12 scale columns fit the 512 TMEM columns; two
// 256-column accumulators would leave none for the scales), 128 K elements
// (four scale blocks) per stage.  Tiles on CTA pairs (cta_group::2, M = 256)
// measured slower than this single-CTA form.  With e4m3 operands for both x
// and W the tiles are 128 x 384 (WIDE): two N = 192 MMAs per K step share the
// x tile, into one 384-column accumulator (measured: issuing every stage's
// MMAs twice took 1.43x the time of once, so with 128 x 192 tiles the tensor
// pipe idled between stages).
// Warp roles: 0 TMA producer (codes every stage, block words every two
// stages, the decoded weights when given), 1 TMEM allocation and the MMA
// issuer (per stage: the tcgen05.cp of the stage's scales into TMEM, then
// four MMAs of K = 32 per N-half that select scale byte j = 0..3), 2-5
// epilogue (2-9 with wide tiles), then the decode warps: codes -> e4m3 bytes
// through an 8-byte per-dialect level table and `prmt`, block words -> scale
// bytes in the tcgen05.cp layout.  With pre-arranged scales (TILES) the
// producer bulk-copies them with the operands and there are no decode warps.
//
// Scale layout (the one tcgen05.cp.32x128b.warpx4 expects): 512 bytes per
// 128 rows, row m's four scale bytes (K-blocks 0..3 of the stage) at
// 16 (m % 32) + 4 (m / 32); the copy replicates them to the four TMEM lane
// quarters, columns 0..3.  B's 192 rows take two such blocks (8 columns).
#pragma once

#include "qs_sd4.cuh"

namespace qs {
namespace sd4 {
namespace gemm_mx {

constexpr int BM = 128, BN = 192, BK = 128;
constexpr int kEpiWarps = 4;
constexpr int kTmemCols = 512;
constexpr int kSfaCol = 2 * BN;      // 4 columns
constexpr int kSfbCol = 2 * BN + 4;  // 8 columns
constexpr int kOpA = BM * BK, kOpB = BN * BK;          // e4m3 tiles, 128-byte rows
constexpr int kSfA = 512, kSfB = 1024;                 // scale bytes of a stage
constexpr int kPkA = BM * BK / 2, kPkB = BN * BK / 2;  // code tiles, 64-byte rows
constexpr int kMetaA = BM * 16, kMetaB = BN * 16;      // 8 block words per row = 2 stages
// Bands of 36 tiles of 192 columns (6912 weight rows; e4m3 x e4m3 at the Wan
// FFN shape: 2.35 ms against 2.53 ms in plain row-major tile order; bands of
// 12 N-tiles 2.39 ms); wide tiles take half as many.
constexpr int kGroupN = 36;
static_assert(BN % 32 == 0 && BN <= 256 && 2 * BN + 12 <= kTmemCols, "tile");

// ADEC / BDEC: the activations / weights come as SD4 codes and are decoded
// to e4m3 in the kernel; otherwise as e4m3 bytes (qs_sd4_quant_e4m3,
// qs_sd4_decode_e4m3) that TMA loads straight into their operand tile.  The
// block words give the scales in every case.
// WIDE (e4m3 x and W only): tiles of 128 x 384, two MMAs of N = 192 per K
// step reading the same x tile, into one 384-column accumulator (the scales
// take 4 + 16 more columns, so a second accumulator does not fit); eight
// epilogue warps, one per TMEM lane quarter and N-half.
// TILES (wide tiles only): the scale bytes come pre-arranged in the
// tensor-memory copy layout (qs_sd4_scale_tiles) and are bulk-copied with the
// operands, so the kernel has no decode warps.
template <bool ADEC, bool BDEC, bool WIDE = false, bool TILES = false>
struct MCfg {
  static_assert(!WIDE || (!ADEC && !BDEC), "wide tiles for e4m3 operands only");
  static_assert(!TILES || WIDE, "pre-arranged scales with wide tiles only");
  static constexpr bool kAnyDec = ADEC || BDEC;
  static constexpr int kHalves = WIDE ? 2 : 1;
  static constexpr int kBN = kHalves * BN;          // tile columns
  static constexpr int kAccBufs = WIDE ? 1 : 2;     // accumulators in tensor memory
  static constexpr int kEpiW = kEpiWarps * kHalves;  // epilogue warps
  static constexpr int kGroup = kGroupN / kHalves;   // N-tiles per band (same columns)
  // decode warps (for e4m3 operands they only turn block words into scale
  // bytes; with wide tiles, 512 rows per stage: 8 warps measured 1.995
  // against 2.148 ms for 4 and 2.020 ms for 16 at the Wan FFN shape)
  static constexpr int kDecWarps = TILES ? 0 : (ADEC ? (BDEC ? 10 : 8) : (WIDE ? 8 : 4));
  static constexpr int kDecThreads = 32 * kDecWarps;
  static constexpr int kThreads = 32 * (2 + kEpiW + kDecWarps);
  // operand stages by measurement (e4m3 x e4m3 at the Wan FFN shape: 3 stages
  // 2.72 ms, 4 stages 2.35 ms, 5 stages 2.47 ms; deeper block-word rings no
  // gain); wide tiles: as many as fit
  static constexpr int kOpStages = (BDEC || WIDE) ? 3 : 4;
  static constexpr int kPkStages = kAnyDec ? kOpStages : 0;
  static constexpr int kMetaSlots = TILES ? 0 : 2;
  static constexpr int kDecRows = (ADEC ? BM : 0) + (BDEC ? BN : 0);  // rows decoded per stage
  static constexpr int kTasks = 2 * kDecRows;  // (row, half of the stage's K)
  static constexpr int kOpStage = kOpA + kHalves * kOpB;
  static constexpr int kSfStage = kSfA + kHalves * kSfB;
  static constexpr int kPkStage = (ADEC ? kPkA : 0) + (BDEC ? kPkB : 0);
  // operand bytes TMA writes straight into an operand stage
  static constexpr int kDirectBytes = (ADEC ? 0 : kOpA) + (BDEC ? 0 : kHalves * kOpB);
  static constexpr int kMetaSlot = kMetaA + kHalves * kMetaB;
  static constexpr int kOffOp = 0;
  static constexpr int kOffSf = kOffOp + kOpStages * kOpStage;
  static constexpr int kOffPk = kOffSf + kOpStages * kSfStage;
  static constexpr int kOffMeta = kOffPk + kPkStages * kPkStage;
  static constexpr int kOffBar = kOffMeta + kMetaSlots * kMetaSlot;
  static constexpr int kNumBars = 2 * kPkStages + 2 * kMetaSlots + 2 * kOpStages + 4;
  static constexpr int kOffEpi = (kOffBar + 8 * kNumBars + 15) / 16 * 16;  // bias of a tile
  static constexpr int kOffTab = kOffEpi + kBN * 4;                         // e4m3 level table
  static constexpr int kOffMisc = kOffTab + kDialects * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  // arrivals completing an operand stage: the decode warps, plus the
  // producer's arm of the direct operands' TMA bytes
  static constexpr int kOpFullCount = kDecWarps + (kDirectBytes ? 1 : 0);
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
  static_assert(kOffSf % 1024 == 0 && kOffPk % 128 == 0 && kOffMeta % 128 == 0, "alignment");
  static_assert(kTasks % (kDecThreads > 0 ? kDecThreads : 1) == 0, "decode split");
  // bytes completing an operand stage by TMA: direct operands and, with
  // TILES, the stage's scale tiles
  static constexpr int kStageTx = kDirectBytes + (TILES ? kSfStage : 0);
  static_assert(!BDEC || ADEC, "codes for W with e4m3 x is not a form of this kernel");
};

// Instruction descriptor of kind::mxf8f6f4.block_scale: e4m3 A and B, both
// K-major, UE8M0 scales, binary32 accumulation; scale byte j of A and B.
__host__ __device__ constexpr uint32_t idesc_mx(int M, int N, uint32_t j) {
  return (j << 4)                                 // B scale byte
         | (0u << 7) | (0u << 10)                 // A, B: E4M3
         | (static_cast<uint32_t>(N >> 3) << 17)  // N / 8
         | (1u << 23)                             // scales: UE8M0
         | (static_cast<uint32_t>(M >> 4) << 24)  // M / 16
         | (j << 29);                             // A scale byte
}

__device__ __forceinline__ void mma_mx(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::
          "r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// Global -> this CTA's shared memory, `bytes` contiguous (16-byte aligned,
// a multiple of 16), completing as transaction bytes on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Shared -> tensor memory: 32 rows of 16 bytes, replicated to the 4 lane quarters.
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// Source descriptor of a 512-byte scale block: no swizzle, K-major, rows of
// 16 bytes, 8-row groups 128 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sf(uint32_t addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr & 0x3FFFFu) >> 4);  // start address
  d |= static_cast<uint64_t>(1) << 16;                  // leading byte offset (one 16-byte unit)
  d |= static_cast<uint64_t>(128 >> 4) << 32;           // stride byte offset
  d |= static_cast<uint64_t>(1) << 46;                  // descriptor version (sm_100)
  return d;                                             // layout type 0: no swizzle
}

// 32 bf16 outputs of one row (pk: 16 packed pairs) as two 16-column pieces,
// each one 32-byte store when `wide` (out 32-byte aligned; rows are 2N bytes
// apart with N % 16 == 0) or two 16-byte stores; `left` = columns to the
// row's end (pieces are whole: N % 16 == 0).
__device__ __forceinline__ void store_row16x2(uint16_t* dst, const uint32_t (&pk)[16], int left,
                                              bool wide) {
#pragma unroll
  for (int v = 0; v < 2; ++v) {
    if (16 * v + 16 > left) break;
    if (wide) {
      asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst + 16 * v),
                   "r"(pk[8 * v]), "r"(pk[8 * v + 1]), "r"(pk[8 * v + 2]), "r"(pk[8 * v + 3]),
                   "r"(pk[8 * v + 4]), "r"(pk[8 * v + 5]), "r"(pk[8 * v + 6]), "r"(pk[8 * v + 7])
                   : "memory");
    } else {
      *reinterpret_cast<uint4*>(dst + 16 * v) =
          make_uint4(pk[8 * v], pk[8 * v + 1], pk[8 * v + 2], pk[8 * v + 3]);
      *reinterpret_cast<uint4*>(dst + 16 * v + 8) =
          make_uint4(pk[8 * v + 4], pk[8 * v + 5], pk[8 * v + 6], pk[8 * v + 7]);
    }
  }
}

struct MBars {
  uint32_t base;
  int P, T, U;  // code stages, meta slots, operand stages
  __device__ uint32_t at(int i) const { return base + 8u * i; }
  __device__ uint32_t pk_full(int s) const { return at(s); }
  __device__ uint32_t pk_empty(int s) const { return at(P + s); }
  __device__ uint32_t meta_full(int s) const { return at(2 * P + s); }
  __device__ uint32_t meta_empty(int s) const { return at(2 * P + T + s); }
  __device__ uint32_t op_full(int s) const { return at(2 * P + 2 * T + s); }
  __device__ uint32_t op_empty(int s) const { return at(2 * P + 2 * T + U + s); }
  __device__ uint32_t acc_full(int b) const { return at(2 * P + 2 * T + 2 * U + b); }
  __device__ uint32_t acc_empty(int b) const { return at(2 * P + 2 * T + 2 * U + 2 + b); }
};

// Tile order: bands of `group` N-tiles of `bn` columns (M-tiles of `bm` rows), every M-tile inside a
// band (N fastest within it), so the tiles the CTAs hold at one time share a
// few MB of activations and weights in L2 and each weight band is read from
// HBM once (kGroupN; see its note).
__device__ __forceinline__ void tile_origin(int t, int m_tiles, int n_tiles, int group, int bm,
                                            int bn, int& m0, int& n0) {
  const int per_group = group * m_tiles;
  const int g = t / per_group, r = t - g * per_group;
  const int gn = min(group, n_tiles - g * group);  // N-tiles in this band
  m0 = (r / gn) * bm;
  n0 = (g * group + r % gn) * bn;
}

// Scale-block offset of row m (within A's 128 rows or B's 192) in a stage.
__device__ __forceinline__ int sf_row_offset(int m) {
  return 512 * (m >> 7) + 16 * (m & 31) + 4 * ((m & 127) >> 5);
}

// out[orow(m)][n] = bf16(fl(sum_k x_hat[m][k] w_hat[n][k]) + bias[n]).  The A
// rows may be longer than the weights' K (kb_wrap K-blocks, walked again):
// the decomposed rows [Q(x) | Q(Delta)] against [w | w].  out_rows (nullable)
// maps accumulator row m to its output row; an index outside [0, out_M) is
// skipped and flagged.
// tmCA / tmCB: the codes (when decoded), tmXA / tmWB: the e4m3 bytes (when
// loaded directly), tmMA / tmMB: the block words; a_tiles / b_tiles: the
// scale tiles (TILES; qs_sd4_scale_tiles layout).
template <bool ADEC, bool BDEC, bool WIDE, bool TILES>
__global__ void __launch_bounds__(MCfg<ADEC, BDEC, WIDE, TILES>::kThreads, 1)
    sd4_mx_gemm_kernel(const __grid_constant__ CUtensorMap tmCA,
                       const __grid_constant__ CUtensorMap tmCB,
                       const __grid_constant__ CUtensorMap tmMA,
                       const __grid_constant__ CUtensorMap tmMB,
                       const __grid_constant__ CUtensorMap tmXA,
                       const __grid_constant__ CUtensorMap tmWB, const uint16_t* __restrict__ bias,
                       uint16_t* __restrict__ out, int M, int N, int K, int kb_wrap,
                       const int32_t* __restrict__ out_rows, int out_M,
                       const uint8_t* __restrict__ a_tiles, const uint8_t* __restrict__ b_tiles) {
  using C = MCfg<ADEC, BDEC, WIDE, TILES>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  uint8_t* sp = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  const MBars bars{sbase + C::kOffBar, C::kPkStages, C::kMetaSlots, C::kOpStages};
  float* epi_b = reinterpret_cast<float*>(sp + C::kOffEpi);
  uint2* tab = reinterpret_cast<uint2*>(sp + C::kOffTab);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sp + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sp + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (N + C::kBN - 1) / C::kBN;
  const int m_tiles = (M + BM - 1) / BM;
  const int num_tiles = m_tiles * n_tiles;
  const int kblocks = K / BK;

  for (int d = threadIdx.x; d < kDialects; d += blockDim.x) {
    uint32_t lo = 0, hi = 0;
    for (int i = 0; i < 4; ++i) {
      lo |= e4m3_eighths(level(d, i)) << (8 * i);
      hi |= e4m3_eighths(level(d, i + 4)) << (8 * i);
    }
    tab[d] = make_uint2(lo, hi);
  }
  // B's scale blocks hold rows 192..255 that no MMA reads but tcgen05.cp copies
  for (int i = threadIdx.x; i < C::kOpStages * C::kSfStage / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(sp + C::kOffSf)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kPkStages; ++s) {
      mbar_init(bars.pk_full(s), 1);
      mbar_init(bars.pk_empty(s), C::kDecWarps);
    }
    for (int s = 0; s < C::kMetaSlots; ++s) {
      mbar_init(bars.meta_full(s), 1);
      mbar_init(bars.meta_empty(s), C::kDecWarps);
    }
    for (int s = 0; s < C::kOpStages; ++s) {
      mbar_init(bars.op_full(s), C::kOpFullCount);
      mbar_init(bars.op_empty(s), 1);
    }
    for (int b = 0; b < C::kAccBufs; ++b) {
      mbar_init(bars.acc_full(b), 1);
      mbar_init(bars.acc_empty(b), C::kEpiW);
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
        int m0, n0;
        tile_origin(t, m_tiles, n_tiles, C::kGroup, BM, C::kBN, m0, n0);
        for (int kb = 0, kbw = 0; kb < kblocks; ++kb, kbw = (kbw + 1 == kb_wrap ? 0 : kbw + 1)) {
          // kbw: the weights' K-block; kb_wrap is even, so both stay in step
          // with the two-stage block-word slots
          if (!TILES && (kb & 1) == 0) {
            if (!mbar_wait_bounded(bars.meta_empty(ms), mph ^ 1u, abort_flag, kErrWaitProducer))
              break;
            const uint32_t dst = sbase + C::kOffMeta + ms * C::kMetaSlot;
            mbar_arrive_expect_tx(bars.meta_full(ms), C::kMetaSlot);
            tma_load_2d(dst, &tmMA, (kb / 2) * 16, m0, bars.meta_full(ms));
#pragma unroll
            for (int h = 0; h < C::kHalves; ++h)
              tma_load_2d(dst + kMetaA + h * kMetaB, &tmMB, (kbw / 2) * 16, n0 + h * BN,
                          bars.meta_full(ms));
            if (++ms == C::kMetaSlots) { ms = 0; mph ^= 1u; }
          }
          if (C::kAnyDec) {  // codes of the decoded operands
            if (!mbar_wait_bounded(bars.pk_empty(s), ph ^ 1u, abort_flag, kErrWaitProducer))
              break;
            const uint32_t dst = sbase + C::kOffPk + s * C::kPkStage;
            mbar_arrive_expect_tx(bars.pk_full(s), C::kPkStage);
            if (ADEC) tma_load_2d(dst, &tmCA, kb * (BK / 2), m0, bars.pk_full(s));
            if (BDEC)
              tma_load_2d(dst + (ADEC ? kPkA : 0), &tmCB, kbw * (BK / 2), n0, bars.pk_full(s));
            if (++s == C::kPkStages) { s = 0; ph ^= 1u; }
          }
          if (C::kDirectBytes) {  // e4m3 operands: TMA into the operand stage
            if (!mbar_wait_bounded(bars.op_empty(so), pho ^ 1u, abort_flag, kErrWaitProducer))
              break;
            const uint32_t ob = sbase + C::kOffOp + so * C::kOpStage;
            mbar_arrive_expect_tx(bars.op_full(so), C::kStageTx);
            if (!ADEC) tma_load_2d(ob, &tmXA, kb * BK, m0, bars.op_full(so));
            if (!BDEC)
#pragma unroll
              for (int h = 0; h < C::kHalves; ++h)
                tma_load_2d(ob + kOpA + h * kOpB, &tmWB, kbw * BK, n0 + h * BN, bars.op_full(so));
            if (TILES) {  // the stage's scale tiles: x rows m0.., W rows n0.. per N-half
              const uint32_t f0 = sbase + C::kOffSf + so * C::kSfStage;
              bulk_load(f0, a_tiles + (static_cast<int64_t>(m0 / BM) * kblocks + kb) * kSfA, kSfA,
                        bars.op_full(so));
#pragma unroll
              for (int h = 0; h < C::kHalves; ++h)
                bulk_load(f0 + kSfA + h * kSfB,
                          b_tiles + (static_cast<int64_t>(n0 / BN + h) * kb_wrap + kbw) * kSfB,
                          kSfB, bars.op_full(so));
            }
            if (++so == C::kOpStages) { so = 0; pho ^= 1u; }
          }
        }
      }
      if (TILES)  // no decode warps: the producer waits for the last releases
        for (int i = 0; i < C::kOpStages; ++i) {
          if (!mbar_wait_bounded(bars.op_empty(so), pho ^ 1u, abort_flag, kErrWaitProducer))
            break;
          if (++so == C::kOpStages) { so = 0; pho ^= 1u; }
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      const uint32_t sfa = tmem_base + kSfaCol, sfb = tmem_base + kSfbCol;
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
        const int buf = it % C::kAccBufs;
        const uint32_t aph = (it / C::kAccBufs) & 1;
        if (!mbar_wait_bounded(bars.acc_empty(buf), aph ^ 1u, abort_flag, kErrWaitMma)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(buf * BN);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_bounded(bars.op_full(s), ph, abort_flag, kErrWaitMma)) break;
          tc_fence_after();
          const uint32_t a0 = sbase + C::kOffOp + s * C::kOpStage;
          const uint32_t b0 = a0 + kOpA;
          const uint32_t f0 = sbase + C::kOffSf + s * C::kSfStage;
          // the stage's scales into TMEM; the tensor pipe runs these copies
          // and the MMAs below in issue order
          tmem_cp_32x128b_x4(sfa, smem_desc_sf(f0));
#pragma unroll
          for (int h = 0; h < C::kHalves; ++h) {  // N-half h: 8 scale columns of its own
            tmem_cp_32x128b_x4(sfb + 8 * h, smem_desc_sf(f0 + kSfA + h * kSfB));
            tmem_cp_32x128b_x4(sfb + 8 * h + 4, smem_desc_sf(f0 + kSfA + h * kSfB + 512));
          }
#pragma unroll
          for (int j = 0; j < BK / 32; ++j)
#pragma unroll
            for (int h = 0; h < C::kHalves; ++h)
              mma_mx(d + h * BN, smem_desc_sw128(a0 + j * 32),
                     smem_desc_sw128(b0 + h * kOpB + j * 32),
                     idesc_mx(BM, BN, static_cast<uint32_t>(j)),
                     sfa + (static_cast<uint32_t>(j) << 30),
                     sfb + 8 * h + (static_cast<uint32_t>(j) << 30), (kb | j) != 0);
          mma_commit(bars.op_empty(s));
          if (++s == C::kOpStages) { s = 0; ph ^= 1u; }
        }
        mma_commit(bars.acc_full(buf));
      }
    }
  } else if (warp < 2 + C::kEpiW) {  // epilogue: TMEM lanes 32 * (warp & 3) ..
    const int quad = warp & 3;
    const int hh = (warp - 2) >> 2;  // N-half of the tile
    const int et = threadIdx.x - 64;
    constexpr int kEpiT = 32 * C::kEpiW;
    int it = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
      const int buf = it % C::kAccBufs;
      const uint32_t aph = (it / C::kAccBufs) & 1;
      int m0, n0;
      tile_origin(t, m_tiles, n_tiles, C::kGroup, BM, C::kBN, m0, n0);
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiT) : "memory");
      for (int i = et; i < C::kBN; i += kEpiT) {
        const int n = n0 + i;
        epi_b[i] = (n < N && bias) ? __uint_as_float(static_cast<uint32_t>(bias[n]) << 16) : 0.f;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiT) : "memory");
      n0 += hh * BN;  // this warp's columns
      const float* e_b = epi_b + hh * BN;
      if (!mbar_wait_bounded(bars.acc_full(buf), aph, abort_flag, kErrWaitEpilogue)) break;
      tc_fence_after();
      const int row = m0 + 32 * quad + lane;
      const bool wide = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
      int orow = row < M ? row : -1;
      if (out_rows && orow >= 0) {
        orow = out_rows[row];
        if (orow < 0 || orow >= out_M) {
          atomicOr(&g_error_word, kErrIndex);
          orow = -1;
        }
      }
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * quad) << 16) +
                             static_cast<uint32_t>(buf * BN + hh * BN);
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
            const float y0 = __fadd_rn(__uint_as_float(r[2 * j]), e_b[32 * c + 2 * j]);
            const float y1 = __fadd_rn(__uint_as_float(r[2 * j + 1]), e_b[32 * c + 2 * j + 1]);
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(y0, y1);
            pk[j] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          uint16_t* dst = out + static_cast<int64_t>(orow) * N + n;
          store_row16x2(dst, pk, N - n, wide);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.acc_empty(buf));
    }
  } else if constexpr (C::kDecWarps > 0) {  // decode warps
    const int dt = threadIdx.x - 32 * (2 + C::kEpiW);  // 0 .. kDecThreads - 1
    int s = 0, so = 0, ms = 0;
    uint32_t ph = 0, pho = 0, mph = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      for (int kb = 0; kb < kblocks; ++kb) {
        if ((kb & 1) == 0 &&
            !mbar_wait_bounded(bars.meta_full(ms), mph, abort_flag, kErrWaitUnpack))
          break;
        if (C::kAnyDec && !mbar_wait_bounded(bars.pk_full(s), ph, abort_flag, kErrWaitUnpack))
          break;
        if (!mbar_wait_bounded(bars.op_empty(so), pho ^ 1u, abort_flag, kErrWaitUnpack)) break;
        const uint8_t* pk = sp + C::kOffPk + s * C::kPkStage;
        const uint8_t* mt = sp + C::kOffMeta + ms * C::kMetaSlot;
        uint8_t* op = sp + C::kOffOp + so * C::kOpStage;
        uint8_t* sf = sp + C::kOffSf + so * C::kSfStage;
        // task = (operand row r: x rows 0..127, then W rows; half h of the
        // stage's K: scale blocks 2h, 2h + 1)
#pragma unroll
        for (int j = 0; j < C::kTasks / C::kDecThreads; ++j) {
          const int task = dt + C::kDecThreads * j;
          const int r = task >> 1, h = task & 1;
          const bool is_b = r >= BM;
          const int rr = is_b ? r - BM : r;
          const uint8_t* crow = pk + (is_b && ADEC ? kPkA : 0) + rr * (BK / 2) + 32 * h;
          const uint32_t words = *reinterpret_cast<const uint32_t*>(
              mt + (is_b ? kMetaA : 0) + rr * 16 + ((kb & 1) * 4 + 2 * h) * 2);
          uint8_t* orow_p = op + (is_b ? kOpA : 0) + rr * 128;
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            // block bb of this half: 16 code bytes (these reads are 2-way
            // bank conflicted; the swizzled stores below are conflict-free,
            // and one order cannot make both free)
            const int bb = b;
            const uint4 cw = *reinterpret_cast<const uint4*>(crow + 16 * bb);
            const uint32_t word = (words >> (16 * bb)) & 0xFFFFu;
            const uint2 E = tab[(word >> 8) & 31u];
            const uint2 o0 = decode8_e4m3(cw.x, E), o1 = decode8_e4m3(cw.y, E);
            const uint2 o2 = decode8_e4m3(cw.z, E), o3 = decode8_e4m3(cw.w, E);
            const int q = 4 * h + 2 * bb;  // 16-byte chunk of the 128-byte row
            *reinterpret_cast<uint4*>(orow_p + ((q ^ (rr & 7)) << 4)) =
                make_uint4(o0.x, o0.y, o1.x, o1.y);
            *reinterpret_cast<uint4*>(orow_p + (((q + 1) ^ (rr & 7)) << 4)) =
                make_uint4(o2.x, o2.y, o3.x, o3.y);
          }
          // the two blocks' UE8M0 scales: e + 127
          const uint32_t e0 = static_cast<uint32_t>(static_cast<int>(static_cast<int8_t>(words & 0xFFu)) + 127);
          const uint32_t e1 = static_cast<uint32_t>(static_cast<int>(static_cast<int8_t>((words >> 16) & 0xFFu)) + 127);
          *reinterpret_cast<uint16_t*>(sf + (is_b ? kSfA : 0) + sf_row_offset(rr) + 2 * h) =
              static_cast<uint16_t>(e0 | (e1 << 8));
        }
        // the scales of the operands loaded as e4m3: one 4-byte word per row
        // (x rows 0..127, then W rows)
        constexpr int kDirectRows = (ADEC ? 0 : BM) + (BDEC ? 0 : C::kBN);
        for (int i = dt; i < kDirectRows; i += C::kDecThreads) {
          const bool is_b = ADEC || i >= BM;
          const int rr = ADEC ? i : (i >= BM ? i - BM : i);  // W rows of both N-halves in turn
          const uint8_t* wp = mt + (is_b ? kMetaA : 0) + rr * 16 + (kb & 1) * 8;
          const uint32_t wv[2] = {*reinterpret_cast<const uint32_t*>(wp),
                                  *reinterpret_cast<const uint32_t*>(wp + 4)};
          uint32_t v = 0;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            v |= static_cast<uint32_t>(
                     static_cast<int>(static_cast<int8_t>((wv[k >> 1] >> (16 * (k & 1))) & 0xFFu)) +
                     127)
                 << (8 * k);
          // W rows: the scale blocks of their N-half (1024 bytes each)
          const int off = is_b ? kSfA + (rr / BN) * kSfB + sf_row_offset(rr % BN)
                               : sf_row_offset(rr);
          *reinterpret_cast<uint32_t*>(sf + off) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bars.op_full(so));
          if (C::kAnyDec) mbar_arrive(bars.pk_empty(s));
          if ((kb & 1) == 1) mbar_arrive(bars.meta_empty(ms));
        }
        if (C::kAnyDec && ++s == C::kPkStages) { s = 0; ph ^= 1u; }
        if (++so == C::kOpStages) { so = 0; pho ^= 1u; }
        if ((kb & 1) == 1 && ++ms == C::kMetaSlots) { ms = 0; mph ^= 1u; }
      }
    }
    // drain: the MMA's last releases of the operand stages have landed
    if (lane == 0)
      for (int i = 0; i < C::kOpStages; ++i) {
        if (!mbar_wait_bounded(bars.op_empty(so), pho ^ 1u, abort_flag, kErrWaitUnpack)) break;
        if (++so == C::kOpStages) { so = 0; pho ^= 1u; }
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

// e4m3 bytes of an SD4 matrix (the magnitudes L/8 with their signs; the
// block words keep the scales): one thread per 16 elements.
__global__ void __launch_bounds__(256) sd4_decode_e4m3_kernel(const uint8_t* __restrict__ codes,
                                                              const uint16_t* __restrict__ meta,
                                                              int64_t rows, int K,
                                                              uint8_t* __restrict__ out) {
  __shared__ uint2 tab[kDialects];
  for (int d = threadIdx.x; d < kDialects; d += blockDim.x) {
    uint32_t lo = 0, hi = 0;
    for (int i = 0; i < 4; ++i) {
      lo |= e4m3_eighths(level(d, i)) << (8 * i);
      hi |= e4m3_eighths(level(d, i + 4)) << (8 * i);
    }
    tab[d] = make_uint2(lo, hi);
  }
  __syncthreads();
  const int64_t per_row = K / 16;
  const int64_t n = rows * per_row;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < n;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = t / per_row;
    const int c = static_cast<int>(t % per_row);
    const uint2 cw = *reinterpret_cast<const uint2*>(codes + row * (K / 2) + c * 8);
    const uint2 E = tab[(meta[row * (K / 32) + c / 2] >> 8) & 31u];
    const uint2 lo = decode8_e4m3(cw.x, E), hi = decode8_e4m3(cw.y, E);
    *reinterpret_cast<uint4*>(out + row * static_cast<int64_t>(K) + c * 16) =
        make_uint4(lo.x, lo.y, hi.x, hi.y);
  }
}

// Scale tiles: the UE8M0 scale bytes (e + 127) of an SD4 matrix, arranged as
// the GEMM copies them into tensor memory, so that one stage's scales are one
// contiguous block for a bulk copy.  Rows go in groups of `group` (BM = 128
// for activations, BN = 192, one N-half, for weights), padded to `slots`
// rows (128 or 256); tile (g, kb) holds slots / 128 blocks of 512 bytes, row
// r of the group and K-block j of the stage at byte sf_row_offset(r) + j.
// Rows past `rows` or past the group's size are zero.  One thread per row
// slot of a tile.
__global__ void __launch_bounds__(256) sd4_scale_tiles_kernel(const uint16_t* __restrict__ meta,
                                                              int64_t rows, int K, int group,
                                                              int slots, int64_t groups,
                                                              uint8_t* __restrict__ tiles) {
  const int kbs = K / BK;
  const int64_t n = groups * kbs * slots;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < n;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int slot = static_cast<int>(t % slots);
    const int64_t gk = t / slots;  // g * kbs + kb
    const int kb = static_cast<int>(gk % kbs);
    const int64_t row = (gk / kbs) * group + slot;
    uint32_t v = 0;
    if (slot < group && row < rows) {
      const uint2 w = *reinterpret_cast<const uint2*>(meta + row * (K / 32) + kb * 4);
      const uint32_t wv[2] = {w.x, w.y};
#pragma unroll
      for (int k = 0; k < 4; ++k)
        v |= static_cast<uint32_t>(
                 static_cast<int>(static_cast<int8_t>((wv[k >> 1] >> (16 * (k & 1))) & 0xFFu)) +
                 127)
             << (8 * k);
    }
    *reinterpret_cast<uint32_t*>(tiles + gk * (slots / 128) * 512 + sf_row_offset(slot)) = v;
  }
}

}  // namespace gemm_mx
}  // namespace sd4
}  // namespace qs
