// DualScale GEMM from pre-quantized codes, one ring of stages.
//
// The same computation as dualscale_gemm_kernel with ASRC_CODES (SegQuant
// DualScale, section "DualScale" of the SegQuant paper: the activation is
// split by sign, q+ and q- codes are multiplied by the int8 weight in two
// products and the two accumulators are folded with their scales), with a
// leaner pipeline:
//   * one stage holds the q+ tile, the q- tile and the weight tile of a k
//     block (3 TMA boxes, one full barrier counting all bytes), and the MMA
//     warp frees it with one tcgen05.commit -- one handshake per k block
//     instead of one per operand ring;
//   * no operand-producer warps: warp 0 issues TMA, warp 1 owns TMEM and
//     issues the MMAs, warps 2.. run the epilogue (8 warps, or 16 when a tile
//     folds several units), which leaves through TMA stores
//     (epilogue_tma_store).
// SINGLE: the single-scale baseline of the same layer (one symmetric scale
// per K segment, s = max|x| / 127 = max(s+, s-)): one code tile per stage,
// one product per k step, one accumulator -- which leaves room for two TMEM
// buffers at every tile width.
// Stage sizes: (2 or 1) x 16 KiB of codes + BN x 128 bytes of weights, as many
// as fit in 224 KiB next to the epilogue's staging tiles (2 or 4 KiB per
// epilogue warp for bf16 or fp32 Y).
// WM (weight mode) 0: int8 weights, one unit per K segment.
// WM 1 (W4): int4 weights with one scale per 128-wide group along K (the SegQuant
// paper's W4A8 setting): TMA brings the packed tile (BN rows of 64 bytes) into
// the stage, two unpack warps widen it to int8 in the 128-byte-swizzled
// layout beside it and signal a per-stage ready barrier that the MMA waits
// on; every k block is its own unit, folded by the epilogue from seeded
// accumulators (epilogue_groups_tma_store, SEED 1).  The seed is written by
// the tensor core: each unit opens with one bf16 MMA, without the old
// accumulator, of a ones column by a seed column (one 8-row swizzle atom
// each, read for every row), which leaves the seed's fp32 bits in every
// accumulator; the int8 MMAs add their int32 sums to those bits.
// WM 2: int8 weight tiles with the units and fp16 scales of int4 groups -- the
// int4 codes rotated by the block Hadamard matrix (HQ-DM, "Single Hadamard
// Transformation", Spanish technical summary 2.1) -- folded from seeded
// accumulators the same way, with the activation scales times the block
// normalization 1/4 (epilogue_groups_tma_store, SEED 2).
#pragma once

#include "gemm_dualscale.cuh"

namespace sq {

constexpr int kCodesEpiWarp0 = 2;

__host__ __device__ constexpr int codes_kernel_threads(bool multi) {
  return (kCodesEpiWarp0 + epi_warps(multi)) * 32;
}
__host__ __device__ constexpr int codes_threads_epw(int epw) { return (kCodesEpiWarp0 + epw) * 32; }

// LDA: the activation code tiles are copied by four loader warps with cp.async
// (16 bytes per thread, eight lanes per 128-byte row, zero-filled past M and
// K) instead of TMA; TMA then carries only the weight tile.  An option (the
// SM's TMA engine moves about 50 bytes per clock in 128-row boxes, less than
// two code tiles plus a weight tile per k block need at the int8 MMA rate),
// measured slower than all-TMA loads on the DiT and MMDiT shapes.
constexpr int kLoaderWarps = 4;
// W4: two int4 unpack warps in the slots after warp 1 (two, not four: with 16
// epilogue warps a block of 20 warps leaves each thread about 96 registers).
constexpr int kUnpackWarps = 2;
__host__ __device__ constexpr int codes_epi_warp0(bool lda, bool w4 = false) {
  return kCodesEpiWarp0 + (lda ? kLoaderWarps : 0) + (w4 ? kUnpackWarps : 0);
}
__host__ __device__ constexpr int codes_threads(int epw, bool lda, bool w4 = false) {
  return (codes_epi_warp0(lda, w4) + epw) * 32;
}

// EPW_: epilogue warps (4, 8 or 16; a multiple of 4, each lane quarter of TMEM
// read by EPW/4 warps splitting the tile's columns).  Four warps let narrow
// tiles (BN = 32, 64, 96) store whole 32-column passes -- the small-M shapes.
// KPS_: k blocks per pipeline stage (1 or 2).  With 2, one full barrier and
// one tcgen05.commit serve two k blocks: the per-stage commit into the ring
// costs the MMA issue stream a few hundred cycles when it comes every k block
// (measured at BN = 128 and 192), much less every second one.  A unit (K
// segment) may begin or end inside a stage.
// Whether two stages of two k blocks fit (with the staging tiles the
// configuration needs): the condition for KPS = 2.
__host__ __device__ constexpr bool codes_kps2_fits(int bn, bool multi, bool y_bf16, bool single,
                                                   int epw) {
  const int stage = 2 * ((single ? 1 : 2) * BM * BK + bn * BK);
  const bool tma_y_forced = single || multi || epw != epi_warps(multi);
  const int y_bytes = epw * stage_y_bytes(y_bf16);
  return (kStageBudget - y_bytes) / stage >= 2 || (!tma_y_forced && kStageBudget / stage >= 2);
}

// STK_ (stacked polarities, one row tile of M <= STK_ rows, one unit per
// tile): the P rows (M rounded up to 16, 32 or 64) are stacked in groups of
// 16 -- group g's q+ box in A rows 32g .. +15, its q- box in rows 32g + 16 ..
// +31 -- so a single MMA per k step yields both products (accumulator lanes
// 32g + r and 32g + 16 + r, both in lane quarter g) and half the MMAs of the
// two-tile form are issued.  The A area of a k block is 2 * STK_ rows; the MMA
// still reads 128 rows from its start (the rows past 2P belong to the weight
// tile or the next k block and land in accumulator lanes nobody reads).
// CSPLIT_ (one row tile: stacked rows, or the two-tile form with four
// epilogue warps): the K range of an N tile is split over the CTAs of a
// cluster; the first CTA keeps an int32 buffer in shared memory -- [2P][BN]
// stacked, [2][128][BN] two-tile -- into which the others add their
// accumulators (bulk reductions by every warp holding accumulator lanes).
// One tile per CTA: one TMEM buffer.
template <int BN_, bool MULTI, bool Y_BF16, bool SINGLE, int EPW_ = epi_warps(MULTI),
          bool LDA_ = false, int KPS_ = 1, int WM_ = 0, int STK_ = 0, bool CSPLIT_ = false>
struct CodesCfg {
  static constexpr bool W4_ = (WM_ == 1);
  static constexpr bool LDA = LDA_;
  static constexpr int KPS = KPS_;
  // full barrier: the TMA thread's arrival (+ bytes), plus one per loader thread
  static constexpr int FULL_COUNT = 1 + (LDA_ ? kLoaderWarps * 32 : 0);
  static constexpr int BN = BN_;
  static constexpr int STK = STK_;
  static constexpr int CODE_TILES = SINGLE ? 1 : 2;    // code boxes per k block
  static constexpr int NACC = (SINGLE || STK_) ? 1 : 2;   // accumulators per unit
  // q+ and q- tiles, or the single code tile, or the stacked rows
  static constexpr int A_BYTES = STK_ ? 2 * STK_ * BK : CODE_TILES * BM * BK;
  static constexpr int W_BYTES = BN * BK;
  static constexpr int WP_BYTES = W4_ ? BN * (BK / 2) : 0;   // packed int4 rows of 64 bytes
  static constexpr int KB_BYTES = A_BYTES + W_BYTES + WP_BYTES;  // one k block of operands
  static constexpr int STAGE = KPS * KB_BYTES;
  static constexpr int EPW = EPW_;
  // Y through TMA stores when two stages still fit beside the staging tiles
  static constexpr bool TMA_Y = SINGLE || MULTI || EPW != epi_warps(MULTI) ||
                                (kStageBudget - EPW * stage_y_bytes(Y_BF16)) / STAGE >= 2;
  static constexpr int Y_BYTES = TMA_Y ? EPW * stage_y_bytes(Y_BF16) : 0;
  // group units: each epilogue warp's two 32-float buffers of widened weight scales
  static constexpr int SW_BYTES = (WM_ != 0) ? EPW * 2 * 32 * 4 : 0;
  // group units: the seed MMA's operands, one 1024-byte swizzle atom each
  static constexpr int SEED_BYTES = (WM_ != 0) ? 2048 : 0;
  // stacked (small M): three stages at most (deeper rings stream no faster);
  // at tiles of up to 64 columns a CTA of the next GEMM in the stream fits on
  // the SM beside this one (shared memory, TMEM and registers) and requests
  // its first weight stages while this one finishes
  static constexpr int S_CAP = STK_ ? 3 : 8;
  // K split: [2P][BN] int32 (stacked) or [2][128][BN] (two-tile form)
  static constexpr int PART_BYTES = CSPLIT_ ? (STK_ ? 2 * STK_ : 2 * BM) * BN_ * 4 : 0;
  static constexpr int S =
      ((kStageBudget - Y_BYTES - SW_BYTES - SEED_BYTES - PART_BYTES) / STAGE) < S_CAP
          ? ((kStageBudget - Y_BYTES - SW_BYTES - SEED_BYTES - PART_BYTES) / STAGE) : S_CAP;
  static_assert(!CSPLIT_ || STK_ != 0 || (!MULTI && !SINGLE && !LDA_ && WM_ == 0 && EPW_ == 4),
                "K split over a cluster: stacked rows, or the two-tile form with four warps");
  static_assert(STK_ == 0 || ((STK_ == 16 || STK_ == 32 || STK_ == 64) && !MULTI && !SINGLE &&
                              !LDA_ && WM_ == 0 && EPW_ == 4),
                "stacked polarities: DualScale, one unit, four epilogue warps");
  static_assert(KPS == 1 || !LDA_, "two k blocks per stage: TMA loads");
  static_assert(WM_ == 0 || (MULTI && !SINGLE && !LDA_ && KPS_ == 1 && BN_ == 128),
                "group units: DualScale, one k block per stage, BN = 128");
  // TMEM accumulator buffers (K split: one tile per CTA, one buffer)
  static constexpr int NBUF = CSPLIT_ ? 1 : ((2 * NACC * BN <= 512) ? 2 : 1);
  // One 256-wide DualScale buffer (both accumulators fill TMEM): the epilogue
  // hands it back in halves, and each tile's first SPLIT_KB k blocks are
  // multiplied into the first half (the first 128 columns of both
  // accumulators) while the previous tile's second half drains, then into
  // the second.
  static constexpr bool SPLIT_DRAIN = BN_ == 256 && NBUF == 1 && NACC == 2 && !MULTI && !SINGLE &&
                                      !LDA_ && KPS_ == 1 && WM_ == 0 && STK_ == 0 && !CSPLIT_ &&
                                      EPW_ == 16 && TMA_Y;   // (the epilogue that releases halves)
  // k blocks multiplied half by half at a tile's start (the rest of the ring
  // keeps loading meanwhile; two or three held their stages through the
  // drain and measured slower)
  static constexpr int SPLIT_KB = 1;
  static constexpr int OFF_Y = S * STAGE;
  static constexpr int OFF_SW = OFF_Y + Y_BYTES;
  static constexpr int OFF_SEED = OFF_SW + SW_BYTES;
  static constexpr int OFF_PART = OFF_SEED + SEED_BYTES;
  static constexpr int OFF_BAR = OFF_PART + PART_BYTES;
  // full, empty; tmem full/empty; drain; (W4) unpacked
  // (+ K split: the partial sums of the other CTAs have landed)
  static constexpr int NUM_BARS = 2 * 8 + 2 * 2 + 1 + (W4_ ? 8 : 0) + (CSPLIT_ ? 1 : 0);
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int TMEM_COLS = NACC * BN * NBUF;
  static constexpr int TMEM_ALLOC = TMEM_COLS <= 256 ? 256 : 512;
  static_assert(S >= 2 && TMEM_COLS <= 512 && SMEM_BYTES <= 232448, "budgets");
  static_assert(BN % 16 == 0 && BN <= 256, "UMMA N for M = 128");
  static_assert(OFF_Y % 1024 == 0 && stage_y_bytes(Y_BF16) % 1024 == 0, "staging alignment");
  static_assert(OFF_SEED % 1024 == 0, "seed atoms: 128-byte swizzle alignment");
  // the MMA's 128-row read from the last k block's A start stays in the allocation
  static_assert(STK_ == 0 || S * STAGE - KB_BYTES + BM * BK <= OFF_MISC, "stacked A read");
};

template <int BN, bool Y_BF16, bool MULTI, bool SINGLE = false, int EPW = epi_warps(MULTI),
          bool LDA = false, int KPS = 1, int WM = 0, int STK = 0, bool CSPLIT = false>
__global__ void __launch_bounds__(codes_threads(EPW, LDA, WM == 1), 1)
    dualscale_gemm_codes_kernel(const __grid_constant__ CUtensorMap tmap_qp,
                                const __grid_constant__ CUtensorMap tmap_qn,
                                const __grid_constant__ CUtensorMap tmap_w,
                                const __grid_constant__ CUtensorMap tmap_y,
                                const __grid_constant__ GemmArgs args) {
  using C = CodesCfg<BN, MULTI, Y_BF16, SINGLE, EPW, LDA, KPS, WM, STK, CSPLIT>;
  constexpr bool W4 = (WM == 1);        // packed int4 tiles, unpack warps
  constexpr bool SEEDED = (WM != 0);    // one unit per k block, seeded accumulators
  constexpr int EPI0 = codes_epi_warp0(LDA, W4);
  static_assert(EPW % 4 == 0 && (BN / (EPW / 4)) % 32 == 0, "32-column store passes per warp");
  static_assert(!MULTI || (BN == 128 && C::NBUF == 2) || (C::NBUF == 1 && BN / (EPW / 4) == 64),
                "several units per tile: BN = 128 with two buffers, or 64 columns per warp");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;                  // [8] codes and weights landed
  uint64_t* empty = full + 8;             // [8] MMAs done with the stage
  uint64_t* tmem_full = empty + 8;        // [2]
  uint64_t* tmem_empty = tmem_full + 2;   // [2]
  uint64_t* drain_bar = tmem_empty + 2;
  uint64_t* ready = drain_bar + 1;        // [8] (W4) int4 tile unpacked
  uint64_t* parts = ready + (W4 ? 8 : 0);  // (K split, first CTA) partial sums added
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long budget = args.wait_budget;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::S; ++i) {
      mbar_init(smem_u32(full + i), C::FULL_COUNT);
      mbar_init(smem_u32(empty + i), 1);
    }
    // (SPLIT_DRAIN: tmem_empty[1] is the first half of the one buffer)
    for (int i = 0; i < (C::SPLIT_DRAIN ? 2 : C::NBUF); ++i) {
      mbar_init(smem_u32(tmem_full + i), 1);
      mbar_init(smem_u32(tmem_empty + i), C::EPW);
    }
    mbar_init(smem_u32(drain_bar), 1);
    if constexpr (W4)
      for (int i = 0; i < C::S; ++i) mbar_init(smem_u32(ready + i), kUnpackWarps);
    if constexpr (CSPLIT) mbar_init(smem_u32(parts), 1);
    *abort_flag = 0;
    fence_mbar_init();
    // K split, first CTA: the others' partial sums arrive as bytes on `parts`
    if constexpr (CSPLIT)
      if (cluster_ctarank() == 0)
        mbar_arrive_expect_tx(smem_u32(parts), (uint32_t)((args.splits - 1) *
                                                          (STK ? 2 * args.a_rows : 2 * BM) * BN * 4));
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_ALLOC);
    tmem_relinquish();
  }
  if constexpr (CSPLIT) {   // the partial-sum buffer starts at zero
    uint4* pb = reinterpret_cast<uint4*>(smem + C::OFF_PART);
    for (int i = threadIdx.x; i < C::PART_BYTES / 16; i += blockDim.x) pb[i] = make_uint4(0, 0, 0, 0);
  }
  if constexpr (SEEDED) {
    // The seed MMA's operands, K-major in the 128-byte swizzle: A (first atom)
    // holds bf16 1.0 and B (second atom) the seed in element 0 of each of its
    // 8 rows -- row r's 16-byte chunk 0 sits at chunk r -- and zeros elsewhere.
    // The seeds are exact in bf16 (their low 16 fp32 bits are zero).
    constexpr uint32_t seed_bits = (WM == 1) ? kMagicW4Bits : kMagicBits;
    static_assert((seed_bits & 0xFFFFu) == 0, "seed exact in bf16");
    uint32_t* sw = reinterpret_cast<uint32_t*>(smem + C::OFF_SEED);
    for (int i = threadIdx.x; i < 512; i += blockDim.x) {
      const int byte = (i & 255) * 4, r = byte >> 7;
      sw[i] = ((byte & 127) == r * 16) ? (i < 256 ? 0x3F80u : (seed_bits >> 16)) : 0u;
    }
    fence_proxy_async_smem();   // read by the tensor core (async proxy)
  }
  tc_fence_before();
  __syncthreads();
  // K split: every CTA of the cluster has its barriers and a zeroed buffer
  // before any of them signals or adds into another's
  if constexpr (CSPLIT) cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_kb = args.num_kb;
  // K split over the cluster: this CTA's k blocks of its cluster's N tile
  const uint32_t crank = CSPLIT ? cluster_ctarank() : 0u;
  // (k blocks shared evenly: every range is nonempty while num_kb >= splits)
  const int kb_lo = CSPLIT ? (int)crank * num_kb / args.splits : 0;
  const int kb_hi = CSPLIT ? ((int)crank + 1) * num_kb / args.splits : num_kb;
  // Setup above overlaps the previous kernel in the stream; what follows the
  // wait reads what earlier kernels wrote (codes, scales) or writes Y.  The
  // next GEMM may start its own setup on SMs this grid leaves free.  (The TMA
  // thread waits after its weight prefetch.)
  grid_dep_launch();
  if (warp != 0) grid_dep_wait();
  const int rounds = CSPLIT ? 1 : num_rounds(args);
  auto tiles = [&](int it, Tile& t) {
    if constexpr (CSPLIT) {   // one N tile per cluster, one row tile
      if (it != 0) return false;
      t.m0 = 0;
      t.n0 = (int)(blockIdx.x / (unsigned)args.splits) * BN;
      t.width = min(BN, args.N - t.n0);
      return true;
    }
    return tile_of(args, it, BN, t);
  };

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_qp);
      if constexpr (!SINGLE) tma_prefetch_desc(&tmap_qn);
      tma_prefetch_desc(&tmap_w);
      tma_prefetch_desc(&tmap_y);
      // bytes one k block brings: the code boxes (a_rows rows each) + the weight box
      const uint32_t kb_tx = (uint32_t)(C::CODE_TILES * (args.a_rows > 0 ? args.a_rows : BM) * BK +
                                        (W4 ? C::WP_BYTES : C::W_BYTES));
      // the q- box: right below the q+ rows (stacked) or its own 128-row tile
      const int qn_off = BM * BK;
      int c = 0;
      bool ok = (args.starve == 0);
      // Stacked (small M): the weight boxes of the first stages are requested
      // before the wait -- no kernel writes the weights -- and their stages'
      // full barriers armed with the whole stage's bytes; the code boxes
      // follow after the wait.
      int pre = 0;
      if constexpr (STK != 0) {
        Tile t0;
        if (ok && tiles(0, t0)) {
          pre = min(C::S, (kb_hi - kb_lo + KPS - 1) / KPS);
          for (int q = 0; q < pre; ++q) {
            const int nk = min(KPS, kb_hi - kb_lo - q * KPS);
            mbar_arrive_expect_tx(smem_u32(full + q), (uint32_t)nk * kb_tx);
            for (int j = 0; j < nk; ++j)
              tma_load_2d(smem_u32(smem + q * C::STAGE + j * C::KB_BYTES + C::A_BYTES), &tmap_w,
                          smem_u32(full + q), (kb_lo + q * KPS + j) * BK, t0.n0);
          }
        }
      }
      grid_dep_wait();
      for (int it = 0; it < rounds && ok; ++it) {
        Tile t;
        if (!tiles(it, t)) continue;
        for (int kb0 = kb_lo; kb0 < kb_hi; kb0 += KPS) {
          const int s = c % C::S;
          const int nk = min(KPS, kb_hi - kb0);            // k blocks in this stage
          const bool prefetched = c < pre;                 // weights already requested
          if (!prefetched) {
            if (!(ok = wait1(smem_u32(empty + s), ((c / C::S) & 1) ^ 1, abort_flag, budget))) break;
            if constexpr (LDA) {
              mbar_arrive_expect_tx(smem_u32(full + s), C::W_BYTES);
            } else {
              mbar_arrive_expect_tx(smem_u32(full + s), (uint32_t)nk * kb_tx);
            }
          }
          for (int j = 0; j < nk; ++j) {
            const int kb = kb0 + j;
            uint8_t* st = smem + s * C::STAGE + j * C::KB_BYTES;
            if constexpr (STK != 0) {   // groups of 16 rows: q+ rows, then q- rows
              if (args.code_box4) {
                const int whole = args.M / 16;   // whole groups: one 4-D box
                if (whole > 0)
                  tma_load_4d(smem_u32(st), &tmap_qp, smem_u32(full + s), kb * BK, 0, 0, t.m0 / 16);
                if (args.code_box4 == 2) {       // the partial group: both planes of its 16 rows
                  tma_load_3d(smem_u32(st + 32 * whole * BK), &tmap_qn, smem_u32(full + s), kb * BK,
                              t.m0 + 16 * whole, 0);
                  tma_load_3d(smem_u32(st + (32 * whole + 16) * BK), &tmap_qn, smem_u32(full + s),
                              kb * BK, t.m0 + 16 * whole, 1);
                }
              } else
              for (int g = 0; g < args.a_rows / 16; ++g) {
                tma_load_2d(smem_u32(st + 32 * g * BK), &tmap_qp, smem_u32(full + s), kb * BK,
                            t.m0 + 16 * g);
                tma_load_2d(smem_u32(st + (32 * g + 16) * BK), &tmap_qn, smem_u32(full + s), kb * BK,
                            t.m0 + 16 * g);
              }
            } else if constexpr (!LDA) {
              tma_load_2d(smem_u32(st), &tmap_qp, smem_u32(full + s), kb * BK, t.m0);
              if constexpr (!SINGLE)
                tma_load_2d(smem_u32(st + qn_off), &tmap_qn, smem_u32(full + s), kb * BK, t.m0);
            }
            if (prefetched) continue;
            if constexpr (W4)   // packed rows land after the unpacked tile's place
              tma_load_2d(smem_u32(st + C::A_BYTES + C::W_BYTES), &tmap_w, smem_u32(full + s),
                          kb * (BK / 2), t.n0);
            else
              tma_load_2d(smem_u32(st + C::A_BYTES), &tmap_w, smem_u32(full + s), kb * BK, t.n0);
          }
          ++c;
        }
      }
      // Let every copy this thread started land before the CTA can exit.
      drain_ring(full, C::S, c, kDrainBudget);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int c = 0, ug = 0;
      bool ok = true;
      for (int it = 0; it < rounds && ok; ++it) {
        Tile t;
        if (!tiles(it, t)) continue;
        const uint32_t idesc = idesc_i8(BM, t.width);
        if constexpr (C::SPLIT_DRAIN && C::SPLIT_KB > 0) {
          // k blocks [kb_lo, kb_lo + P) into the first half as soon as it is
          // free, then into the second half once the whole buffer is; the
          // rest at full width.  Their stages are released after both halves.
          const int P = min(min(C::SPLIT_KB, C::S), kb_hi - kb_lo);
          const uint32_t par = (ug & 1) ^ 1;
          const uint32_t d = tmem_base;
          const int w1 = t.width - 128;                      // second half's columns
          auto half = [&](int q, int col, uint32_t hdesc) {
            const int s = (c + q) % C::S;
            const uint32_t a_p = smem_u32(smem + s * C::STAGE);
            const uint32_t a_n = a_p + BM * BK;
            const uint32_t b_w = a_p + C::A_BYTES + (uint32_t)col * BK;   // weight rows col ..
#pragma unroll
            for (int ks = 0; ks < BK / 32; ++ks) {
              const uint32_t acc = (q > 0 || ks > 0) ? 1u : 0u;
              const uint64_t bd = smem_desc_k_sw128(b_w + ks * 32);
              umma_i8(d + (uint32_t)col, smem_desc_k_sw128(a_p + ks * 32), bd, hdesc, acc);
              umma_i8(d + BN + (uint32_t)col, smem_desc_k_sw128(a_n + ks * 32), bd, hdesc, acc);
            }
          };
          if (!(ok = wait1(smem_u32(tmem_empty + 1), par, abort_flag, budget))) break;
          tc_fence_after();
          for (int q = 0; q < P; ++q) {
            if (!(ok = wait1(smem_u32(full + (c + q) % C::S), ((c + q) / C::S) & 1, abort_flag,
                             budget)))
              break;
            half(q, 0, idesc_i8(BM, min(t.width, 128)));
          }
          if (!ok) break;
          if (!(ok = wait1(smem_u32(tmem_empty), par, abort_flag, budget))) break;
          tc_fence_after();
          for (int q = 0; q < P; ++q) {
            if (w1 > 0) half(q, 128, idesc_i8(BM, w1));
            umma_commit(smem_u32(empty + (c + q) % C::S));
          }
          c += P;
          for (int kb = kb_lo + P; kb < kb_hi; ++kb) {
            const int s = c % C::S;
            if (!(ok = wait1(smem_u32(full + s), (c / C::S) & 1, abort_flag, budget))) break;
            const uint32_t a_p = smem_u32(smem + s * C::STAGE);
            const uint32_t a_n = a_p + BM * BK;
            const uint32_t b_w = a_p + C::A_BYTES;
#pragma unroll
            for (int ks = 0; ks < BK / 32; ++ks) {
              const uint64_t bd = smem_desc_k_sw128(b_w + ks * 32);
              umma_i8(d, smem_desc_k_sw128(a_p + ks * 32), bd, idesc, 1u);
              umma_i8(d + BN, smem_desc_k_sw128(a_n + ks * 32), bd, idesc, 1u);
            }
            umma_commit(smem_u32(empty + s));
            ++c;
          }
          if (!ok) break;
          umma_commit(smem_u32(tmem_full));
          ++ug;
          continue;
        }
        bool unit_open = false;
        uint32_t d_pos = 0;
        for (int kb0 = kb_lo; kb0 < kb_hi && ok; kb0 += KPS) {
          const int s = c % C::S;
          // W4: the unpack warps' ready barrier (it follows the stage's full barrier)
          if (!(ok = wait1(smem_u32((W4 ? ready : full) + s), (c / C::S) & 1, abort_flag, budget))) break;
          // tiles written by cp.async or by the unpack warps (generic proxy)
          // before the tensor core reads them
          if constexpr (LDA || W4) fence_proxy_async_smem();
          const int nk = min(KPS, kb_hi - kb0);
          for (int j = 0; j < nk; ++j) {
            const int kb = kb0 + j;
            if (!unit_open) {   // a unit (K segment) may start inside a stage
              const int b = ug % C::NBUF;
              const uint32_t par = ((ug / C::NBUF) & 1) ^ 1;
              if (!(ok = wait1(smem_u32(tmem_empty + b), par, abort_flag, budget))) break;
              tc_fence_after();
              d_pos = tmem_base + (uint32_t)(b * C::NACC * BN);
              // group units: both accumulators set to the seed's bits (1 x seed, fp32)
              if constexpr (SEEDED)
                umma_bf16(d_pos, smem_desc_k_sw128_atom(smem_u32(smem + C::OFF_SEED)),
                          smem_desc_k_sw128_atom(smem_u32(smem + C::OFF_SEED + 1024)),
                          idesc_bf16(BM, C::NACC * BN), 0u);
            }
            const uint32_t a_p = smem_u32(smem + s * C::STAGE + j * C::KB_BYTES);
            const uint32_t a_n = a_p + BM * BK;
            const uint32_t b_w = a_p + C::A_BYTES;
#pragma unroll
            for (int ks = 0; ks < BK / 32; ++ks) {
              const uint32_t acc = (SEEDED || unit_open || ks > 0) ? 1u : 0u;
              const uint64_t bd = smem_desc_k_sw128(b_w + ks * 32);
              umma_i8(d_pos, smem_desc_k_sw128(a_p + ks * 32), bd, idesc, acc);
              if constexpr (!SINGLE && !STK)
                umma_i8(d_pos + BN, smem_desc_k_sw128(a_n + ks * 32), bd, idesc, acc);
            }
            unit_open = true;
            // (K split: the CTA's range is one unit)
            if (CSPLIT ? kb + 1 == kb_hi : kb_closes_unit(args, kb)) {
              umma_commit(smem_u32(tmem_full + (ug % C::NBUF)));
              ++ug;
              unit_open = false;
            }
          }
          if (!ok) break;
          umma_commit(smem_u32(empty + s));
          ++c;
        }
      }
      // All MMAs this thread issued have landed once the drain barrier flips.
      umma_commit(smem_u32(drain_bar));
      wait_drain(smem_u32(drain_bar), 0, kDrainBudget);
    }
  } else if (warp < EPI0) {
    // --------------------------------------------- code-tile loader warps (LDA)
    // Thread t: rows (t >> 5) * 32 + 4 * i + ((t & 31) >> 3), i = 0..7, 16-byte
    // chunk t & 7 of the row's 128-byte k block, stored at the 128-byte-swizzle
    // position (chunk ^ (row & 7)) of the row -- the layout TMA would write.
    if constexpr (LDA) {
      const int t_id = threadIdx.x - kCodesEpiWarp0 * 32;   // 0..127
      const int chunk = t_id & 7;
      const int r0 = (t_id >> 5) * 32 + ((t_id & 31) >> 3);
      int c = 0;
      bool ok = (args.starve == 0);
      for (int it = 0; it < rounds && ok; ++it) {
        Tile t;
        if (!tiles(it, t)) continue;
        for (int kb = 0; kb < num_kb; ++kb) {
          const int s = c % C::S;
          if (!(ok = wait_warp(smem_u32(empty + s), ((c / C::S) & 1) ^ 1, abort_flag, budget))) break;
          const uint32_t st = smem_u32(smem + s * C::STAGE);
          const int k = kb * BK + chunk * 16;
          const bool k_in = k < args.K;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = r0 + 4 * i;
            const int grow = t.m0 + r;
            const bool in = k_in && grow < args.M;
            const int64_t off = in ? (int64_t)grow * args.lda + k : 0;
            const uint32_t dst = st + (uint32_t)(r * 128 + ((chunk ^ (r & 7)) << 4));
            cp_async16(dst, args.a_pos + off, in ? 16u : 0u);
            if constexpr (!SINGLE) cp_async16(dst + BM * BK, args.a_neg + off, in ? 16u : 0u);
          }
          cp_async_arrive_noinc(smem_u32(full + s));
          ++c;
        }
      }
      // every copy of this thread has landed before the CTA can exit
      asm volatile("cp.async.wait_all;" ::: "memory");
    } else if constexpr (W4) {
      // int4 unpack: thread t widens 16-byte pieces task = i*64 + t of the
      // packed tile (row n = task / 4, quarter q = task % 4: 32 codes, low
      // nibble first) into two 16-byte chunks of the int8 row at their
      // 128-byte-swizzle positions, each byte 16 x its code (the epilogue's
      // accumulator seed accounts for the factor).
      const int t_id = threadIdx.x - kCodesEpiWarp0 * 32;   // 0..63
      int c = 0;
      bool ok = (args.starve == 0);
      for (int it = 0; it < rounds && ok; ++it) {
        Tile t;
        if (!tiles(it, t)) continue;
        for (int kb = 0; kb < num_kb; ++kb) {
          const int s = c % C::S;
          if (!(ok = wait_warp(smem_u32(full + s), (c / C::S) & 1, abort_flag, budget))) break;
          uint8_t* st = smem + s * C::STAGE;
          const uint8_t* src = st + C::A_BYTES + C::W_BYTES;
          uint8_t* dst = st + C::A_BYTES;
#pragma unroll
          for (int i = 0; i < (BN * 4) / (kUnpackWarps * 32); ++i) {
            const int task = i * (kUnpackWarps * 32) + t_id;
            const int n = task >> 2, q = task & 3;
            const uint4 pk = *reinterpret_cast<const uint4*>(src + n * 64 + q * 16);
            const uint2 e0 = unpack8_int4_x16(pk.x), e1 = unpack8_int4_x16(pk.y);
            const uint2 e2 = unpack8_int4_x16(pk.z), e3 = unpack8_int4_x16(pk.w);
            uint8_t* drow = dst + n * 128;
            *reinterpret_cast<uint4*>(drow + (((2 * q) ^ (n & 7)) << 4)) = make_uint4(e0.x, e0.y, e1.x, e1.y);
            *reinterpret_cast<uint4*>(drow + (((2 * q + 1) ^ (n & 7)) << 4)) = make_uint4(e2.x, e2.y, e3.x, e3.y);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(ready + s));
          ++c;
        }
      }
    }
  } else {
    // --------------------------------------------------------- epilogue
    // Warp w reads TMEM lanes 32*(w % 4) .. +31; the EPW epilogue warps cover
    // each lane quarter once per column part.
    const int quad = warp & 3;
    const int part = (warp - EPI0) >> 2;
    const uint32_t t_lane = tmem_base + ((uint32_t)(quad * 32) << 16);
    if constexpr (STK != 0) {
      static_assert(!STK || C::Y_BYTES == 4 * stage_y_bytes(Y_BF16), "four staging tiles");
      epilogue_stacked<BN, C::NBUF, Y_BF16, CSPLIT>(
          args, &tmap_y, smem + C::OFF_Y, quad, lane, t_lane, tmem_full, smem_u32(tmem_empty), rounds,
          tiles, abort_flag, budget, crank, smem_u32(smem + C::OFF_PART), smem_u32(parts));
    } else if constexpr (SEEDED) {
      uint8_t* stage_y = smem + C::OFF_Y + (warp - EPI0) * stage_y_bytes(Y_BF16);
      float* sw_stage = reinterpret_cast<float*>(smem + C::OFF_SW) + (warp - EPI0) * 64;
      epilogue_groups_tma_store<C::EPW, Y_BF16, WM>(
          args, &tmap_y, stage_y, sw_stage, quad, part, lane, t_lane, tmem_full,
          smem_u32(tmem_empty), rounds, tiles, abort_flag, budget);
    } else if constexpr (C::TMA_Y) {
      uint8_t* stage_y = smem + C::OFF_Y + (warp - EPI0) * stage_y_bytes(Y_BF16);
      epilogue_tma_store<BN, C::NBUF, C::EPW, C::NACC, MULTI, Y_BF16, decltype(tiles), false, CSPLIT,
                         C::SPLIT_DRAIN>(
          args, &tmap_y, stage_y, quad, part, lane, t_lane, tmem_full, smem_u32(tmem_empty), rounds,
          tiles, abort_flag, budget, 0, false, crank, smem_u32(smem + C::OFF_PART), smem_u32(parts));
    } else {
      // no room for staging tiles: 16-byte stores straight from registers (DualScale, one unit)
      epilogue_role<BN, C::NBUF, false, false, Y_BF16, false>(
          args, quad, part, lane, t_lane, tmem_full, smem_u32(tmem_empty), /*empty_remote=*/false,
          /*row_shift=*/0, rounds, tiles, abort_flag, budget);
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  // K split: the first CTA's buffer outlives every add into it.  Without an
  // abort its epilogue has already seen every byte on `parts`; after one, the
  // other CTAs still send their slices, so it waits for them here (bounded)
  // while the others wait at the cluster barrier.
  if constexpr (CSPLIT) {
    if (threadIdx.x == 0 && crank == 0 && *abort_flag) wait_drain(smem_u32(parts), 0, 2 * budget);
    cluster_sync();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_ALLOC);
  }
}

}  // namespace sq
