// DualScale GEMM from pre-quantized codes on CTA pairs (2-SM UMMA, sm_100a).
//
// Same computation as dualscale_gemm_kernel with ASRC_CODES and int8 weights
// (SegQuant DualScale: two int8 products per unit fused in the epilogue; see
// gemm_dualscale.cuh), issued as tcgen05.mma.cta_group::2: a pair tile is 256
// token rows (128 per CTA) by BN output columns, and each CTA loads only half
// of the weight tile, so every weight byte in shared memory feeds twice the
// MMA work of the one-CTA kernel.
//
// Per CTA of the pair:
//   * warp 0: TMA of its 128 rows of q+ / q- and its BN/2 weight rows into one
//     stage, once its own `empty` barrier says the pair's MMAs are done with
//     the stage.  All copies of a stage complete on the leader's `full`
//     barrier, which the leader arms with both CTAs' bytes; a peer copy that
//     lands before the leader armed the barrier only takes its transaction
//     count below zero for a while (the phase still needs the leader's
//     arrival);
//   * warp 1: TMEM allocation for the pair; in the leader (rank 0) the single
//     MMA-issuing thread;
//   * warps 2..: epilogue (epilogue_tma_store): read this CTA's 128 TMEM lanes,
//     fold, stage and store its rows with TMA stores, and arrive on the
//     leader's `tmem_empty` barrier as soon as the last TMEM loads landed.
// Per SM and k block the pair moves 32 KiB of codes and BN/2 x 128 bytes of
// weights, and its tensor core reads only its own half of the weight tile:
// at BN = 256 that is 48 KiB and half the shared-memory operand traffic of
// the one-CTA 256-wide tile.
// The leader commits the MMAs of every KP consecutive stages to both CTAs'
// `empty` barrier of that stage group, and each unit to both CTAs'
// `tmem_full` barriers, each with one multicast commit.
#pragma once

#include "gemm_dualscale.cuh"

namespace sq {

constexpr int BM_PAIR = 2 * BM;  // token rows per pair tile

constexpr int kPairEpiWarp0 = 2;
__host__ __device__ constexpr int pair_threads(int epw) { return (kPairEpiWarp0 + epw) * 32; }

template <int BN_, int EPW_, bool Y_BF16>
struct PairCfg {
  static constexpr int BN = BN_;
  static constexpr int EPW = EPW_;
  static constexpr int HB = BN / 2;                 // weight rows loaded per CTA
  static constexpr int Q_TILE = BM * BK;
  static constexpr int W_HALF = HB * BK;
  static constexpr int STAGE = 2 * Q_TILE + W_HALF;
  static constexpr int Y_BYTES = EPW * stage_y_bytes(Y_BF16);
  static constexpr int S = ((kStageBudget - Y_BYTES) / STAGE) < 8 ? ((kStageBudget - Y_BYTES) / STAGE) : 8;
  // stages per release of the ring: one (releasing two at a time measured
  // slower with the four stages that fit: 705 against 693 us on the MMDiT shape)
  static constexpr int KP = 1;
  static constexpr int NBUF = (BN <= 128) ? 2 : 1;
  static constexpr int OFF_Y = S * STAGE;
  static constexpr int OFF_BAR = OFF_Y + Y_BYTES;
  static constexpr int NUM_BARS = 2 * 8 + 2 * 2 + 1;  // full, empty; tmem full/empty; drain
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int TMEM_COLS = 2 * BN * NBUF;
  static constexpr int TMEM_ALLOC = TMEM_COLS <= 256 ? 256 : 512;
  static_assert(BN % 32 == 0 && BN <= 256, "pair UMMA N");
  static_assert(S >= 2 && TMEM_COLS <= 512 && SMEM_BYTES <= 232448, "budgets");
  static_assert(OFF_Y % 1024 == 0, "staging alignment");
};

// Pair tiles in the same snake order as tile_of, over pairs of CTAs; m_tiles
// counts 256-row tiles.
__device__ __forceinline__ bool pair_tile_of(const GemmArgs& a, int it, int bn, Tile& t) {
  const int npairs = gridDim.x >> 1, pair = blockIdx.x >> 1;
  const int pos = (it & 1) ? (npairs - 1 - pair) : pair;
  const int idx = it * npairs + pos;
  if (idx >= a.num_tiles) return false;
  const int nfull_tiles = a.m_tiles * a.n_full;
  if (idx < nfull_tiles) {
    t.m0 = (idx / a.n_full) * BM_PAIR;
    t.n0 = (idx % a.n_full) * bn;
    t.width = bn;
  } else {
    t.m0 = (idx - nfull_tiles) * BM_PAIR;
    t.n0 = a.n_full * bn;
    t.width = a.tail;
  }
  return true;
}

template <int BN, bool Y_BF16, bool MULTI, int EPW>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair_threads(EPW), 1)
    dualscale_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_qp,
                               const __grid_constant__ CUtensorMap tmap_qn,
                               const __grid_constant__ CUtensorMap tmap_w,
                               const __grid_constant__ CUtensorMap tmap_y,
                               const __grid_constant__ GemmArgs args) {
  using C = PairCfg<BN, EPW, Y_BF16>;
  static_assert(EPW % 4 == 0 && (BN / (EPW / 4)) % 32 == 0, "32-column store passes per warp");
  static_assert(!MULTI || BN / (EPW / 4) <= 64, "several units: at most 64 partials per thread");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;              // [8] (leader) both CTAs' copies landed
  uint64_t* empty = full + 8;         // [8 / KP] (both) the pair's MMAs are done with the stages
  uint64_t* tmem_full = empty + 8;    // [2]
  uint64_t* tmem_empty = tmem_full + 2;  // [2] (leader) both CTAs drained the buffer
  uint64_t* drain_bar = tmem_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const long long budget = args.wait_budget;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::S; ++i) mbar_init(smem_u32(full + i), 1);
    for (int i = 0; i < C::S / C::KP; ++i) mbar_init(smem_u32(empty + i), 1);
    for (int i = 0; i < C::NBUF; ++i) {
      mbar_init(smem_u32(tmem_full + i), 1);
      mbar_init(smem_u32(tmem_empty + i), 2 * EPW);
    }
    mbar_init(smem_u32(drain_bar), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), C::TMEM_ALLOC);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  // Both CTAs' barriers exist before either signals the other.
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_kb = args.num_kb;
  const int rounds = (args.num_tiles + (int)(gridDim.x >> 1) - 1) / (int)(gridDim.x >> 1);
  auto tiles = [&](int it, Tile& t) { return pair_tile_of(args, it, BN, t); };

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_qp);
      tma_prefetch_desc(&tmap_qn);
      tma_prefetch_desc(&tmap_w);
      tma_prefetch_desc(&tmap_y);
      const uint32_t full0 = mapa_shared(smem_u32(full), 0);   // leader's barriers
      int c = 0;
      bool ok = (args.starve == 0);
      for (int it = 0; it < rounds && ok; ++it) {
        Tile t;
        if (!tiles(it, t)) continue;
        const int m_cta = t.m0 + (int)rank * BM;
        const int n_cta = t.n0 + (int)rank * (t.width / 2);
        for (int kb = 0; kb < num_kb; ++kb) {
          const int s = c % C::S;
          if (s % C::KP == 0 &&
              !(ok = wait1s<true>(smem_u32(empty + s / C::KP), ((c / C::S) & 1) ^ 1, abort_flag,
                                  budget)))
            break;
          if (leader) mbar_arrive_expect_tx(smem_u32(full + s), 2 * C::STAGE);
          uint8_t* st = smem + s * C::STAGE;
          const uint32_t bar = full0 + 8u * (uint32_t)s;
          tma_load_2d_pair(smem_u32(st), &tmap_qp, bar, kb * BK, m_cta);
          tma_load_2d_pair(smem_u32(st + C::Q_TILE), &tmap_qn, bar, kb * BK, m_cta);
          tma_load_2d_pair(smem_u32(st + 2 * C::Q_TILE), &tmap_w, bar, kb * BK, n_cta);
          ++c;
        }
      }
      // The leader's `full` phases count both CTAs' copies: draining them lets
      // every issued copy land before the pair tears down (the cluster barrier
      // of the teardown holds the peer until then).
      if (leader) drain_ring(full, C::S, c, kDrainBudget);
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------- MMA issuer (pair)
      int c = 0, ug = 0;
      bool ok = true;
      for (int it = 0; it < rounds && ok; ++it) {
        Tile t;
        if (!tiles(it, t)) continue;
        const uint32_t idesc = idesc_i8(BM_PAIR, t.width);
        bool unit_open = false;
        uint32_t d_pos = 0;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!unit_open) {
            const int b = ug % C::NBUF;
            if (!(ok = wait1s<true>(smem_u32(tmem_empty + b), ((ug / C::NBUF) & 1) ^ 1, abort_flag, budget)))
              break;
            tc_fence_after();
            d_pos = tmem_base + (uint32_t)(b * 2 * BN);
          }
          const int s = c % C::S;
          const uint32_t par = (c / C::S) & 1;
          if (!(ok = wait1s<true>(smem_u32(full + s), par, abort_flag, budget))) break;
          tc_fence_after();
          const uint32_t a_p = smem_u32(smem + s * C::STAGE);
          const uint32_t a_n = a_p + C::Q_TILE;
          const uint32_t b_w = a_p + 2 * C::Q_TILE;
#pragma unroll
          for (int ks = 0; ks < BK / 32; ++ks) {
            const uint32_t acc = (unit_open || ks > 0) ? 1u : 0u;
            const uint64_t bd = smem_desc_k_sw128(b_w + ks * 32);
            umma_i8_pair(d_pos, smem_desc_k_sw128(a_p + ks * 32), bd, idesc, acc);
            umma_i8_pair(d_pos + BN, smem_desc_k_sw128(a_n + ks * 32), bd, idesc, acc);
          }
          unit_open = true;
          if (s % C::KP == C::KP - 1) umma_commit_pair_to(smem_u32(empty + s / C::KP), 0x3);
          ++c;
          if (kb_closes_unit(args, kb)) {
            umma_commit_pair_to(smem_u32(tmem_full + ug % C::NBUF), 0x3);
            ++ug;
            unit_open = false;
          }
        }
      }
      umma_commit_pair(smem_u32(drain_bar));
      wait_drain(smem_u32(drain_bar), 0, kDrainBudget);
    }
  } else if (warp >= kPairEpiWarp0) {
    // --------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int part = (warp - kPairEpiWarp0) >> 2;
    const uint32_t empty0 = smem_u32(tmem_empty);
    uint8_t* stage_y = smem + C::OFF_Y + (warp - kPairEpiWarp0) * stage_y_bytes(Y_BF16);
    epilogue_tma_store<BN, C::NBUF, EPW, 2, MULTI, Y_BF16, decltype(tiles), true>(
        args, &tmap_y, stage_y, quad, part, lane, tmem_base + ((uint32_t)(quad * 32) << 16),
        tmem_full, leader ? empty0 : mapa_shared(empty0, 0), rounds, tiles, abort_flag, budget,
        (int)rank * BM, /*empty_remote=*/!leader);
  }

  // ---------------------------------------------------------------- teardown
  // The leader's MMAs read the peer's shared memory and write its TMEM, and the
  // peer signals the leader's barriers: neither CTA frees TMEM or exits before
  // both have finished.
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_ALLOC);
  }
}

}  // namespace sq
