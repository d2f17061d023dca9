// DualScale GEMM from combined codes c = q+ + q- (one signed byte per
// activation).
//
// SegQuant DualScale (section "DualScale" of the SegQuant paper) splits the
// activation by sign; the two parts have disjoint support, so the pair
// (q+, q-) is carried losslessly by c: q+ = max(c, 0), q- = min(c, 0).  The
// codes therefore cross HBM and L2 once, at one byte per activation, and the
// kernel splits each tile in shared memory before the two int8 products.
//
// Pipeline (one ring of stages): warp 0 loads the c tile (16 KiB) into the
// first half of the stage's 32 KiB activation area and the weight tile after
// it; splitter warps 2..5 (thread r owns tile row r) read the row's eight
// swizzled 16-byte chunks, write q+ over them and q- to the same chunk
// positions of the second half (both halves are 1024-byte aligned, so the
// 128-byte swizzle maps a (row, chunk) pair to the same offset in each), then
// signal `ready`; warp 1 issues the MMAs on q+ / q- and frees the stage with
// one commit; epilogue warps 6.. fold and store.  A row is rewritten only by
// the thread that has already read it, so no barrier between threads is
// needed.
#pragma once

#include "gemm_dualscale.cuh"

namespace sq {

constexpr int kCombSplitWarp0 = 2;
constexpr int kCombSplitWarps = 4;   // BM rows / 32
constexpr int kCombEpiWarp0 = kCombSplitWarp0 + kCombSplitWarps;   // 6

__host__ __device__ constexpr int combined_kernel_threads(bool multi) {
  return (kCombEpiWarp0 + epi_warps(multi)) * 32;
}

template <int BN_>
struct CombinedCfg {
  static constexpr int BN = BN_;
  static constexpr int C_BYTES = BM * BK;            // the c tile as loaded
  static constexpr int A_BYTES = 2 * BM * BK;        // q+ tile, q- tile after the split
  static constexpr int W_BYTES = BN * BK;
  static constexpr int STAGE = A_BYTES + W_BYTES;
  static constexpr int TX_BYTES = C_BYTES + W_BYTES; // bytes TMA writes per stage
  static constexpr int S = (kStageBudget / STAGE) < 8 ? (kStageBudget / STAGE) : 8;
  static constexpr int NBUF = (BN <= 128) ? 2 : 1;
  static constexpr int OFF_BAR = S * STAGE;
  static constexpr int NUM_BARS = 3 * 8 + 2 * 2 + 1;  // full, ready, empty; tmem full/empty; drain
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int TMEM_COLS = 2 * BN * NBUF;
  static constexpr int TMEM_ALLOC = TMEM_COLS <= 256 ? 256 : 512;
  static_assert(S >= 2 && TMEM_COLS <= 512 && SMEM_BYTES <= 232448, "budgets");
  static_assert(BN % 16 == 0 && BN <= 256, "UMMA N for M = 128");
  static_assert(BM == kCombSplitWarps * 32, "one splitter thread per tile row");
};

template <int BN, bool Y_BF16, bool MULTI>
__global__ void __launch_bounds__(combined_kernel_threads(MULTI), 1)
    dualscale_gemm_combined_kernel(const __grid_constant__ CUtensorMap tmap_c,
                                   const __grid_constant__ CUtensorMap tmap_w,
                                   const __grid_constant__ GemmArgs args) {
  using C = CombinedCfg<BN>;
  static_assert(!MULTI || BN == 128, "several units per tile need double-buffered TMEM");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;                  // [8] c and weights landed
  uint64_t* ready = full + 8;             // [8] q+ / q- written
  uint64_t* empty = ready + 8;            // [8] MMAs done with the stage
  uint64_t* tmem_full = empty + 8;        // [2]
  uint64_t* tmem_empty = tmem_full + 2;   // [2]
  uint64_t* drain_bar = tmem_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long budget = args.wait_budget;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::S; ++i) {
      mbar_init(smem_u32(full + i), 1);
      mbar_init(smem_u32(ready + i), kCombSplitWarps);
      mbar_init(smem_u32(empty + i), 1);
    }
    for (int i = 0; i < C::NBUF; ++i) {
      mbar_init(smem_u32(tmem_full + i), 1);
      mbar_init(smem_u32(tmem_empty + i), epi_warps(MULTI));
    }
    mbar_init(smem_u32(drain_bar), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_ALLOC);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_kb = args.num_kb;
  const int rounds = num_rounds(args);
  auto tiles = [&](int it, Tile& t) { return tile_of(args, it, BN, t); };

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_c);
      tma_prefetch_desc(&tmap_w);
      int c = 0;
      bool ok = (args.starve == 0);
      for (int it = 0; it < rounds && ok; ++it) {
        Tile t;
        if (!tiles(it, t)) continue;
        for (int kb = 0; kb < num_kb; ++kb) {
          const int s = c % C::S;
          if (!(ok = wait1(smem_u32(empty + s), ((c / C::S) & 1) ^ 1, abort_flag, budget))) break;
          uint8_t* st = smem + s * C::STAGE;
          mbar_arrive_expect_tx(smem_u32(full + s), C::TX_BYTES);
          tma_load_2d(smem_u32(st), &tmap_c, smem_u32(full + s), kb * BK, t.m0);
          tma_load_2d(smem_u32(st + C::A_BYTES), &tmap_w, smem_u32(full + s), kb * BK, t.n0);
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
        bool unit_open = false;
        uint32_t d_pos = 0;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!unit_open) {
            const int b = ug % C::NBUF;
            if (!(ok = wait1(smem_u32(tmem_empty + b), ((ug / C::NBUF) & 1) ^ 1, abort_flag, budget))) break;
            tc_fence_after();
            d_pos = tmem_base + (uint32_t)(b * 2 * BN);
          }
          const int s = c % C::S;
          if (!(ok = wait1(smem_u32(ready + s), (c / C::S) & 1, abort_flag, budget))) break;
          tc_fence_after();
          const uint32_t a_p = smem_u32(smem + s * C::STAGE);
          const uint32_t a_n = a_p + C::C_BYTES;
          const uint32_t b_w = a_p + C::A_BYTES;
#pragma unroll
          for (int ks = 0; ks < BK / 32; ++ks) {
            const uint32_t acc = (unit_open || ks > 0) ? 1u : 0u;
            const uint64_t bd = smem_desc_k_sw128(b_w + ks * 32);
            umma_i8(d_pos, smem_desc_k_sw128(a_p + ks * 32), bd, idesc, acc);
            umma_i8(d_pos + BN, smem_desc_k_sw128(a_n + ks * 32), bd, idesc, acc);
          }
          unit_open = true;
          umma_commit(smem_u32(empty + s));
          ++c;
          if (kb_closes_unit(args, kb)) {
            umma_commit(smem_u32(tmem_full + (ug % C::NBUF)));
            ++ug;
            unit_open = false;
          }
        }
      }
      // All MMAs this thread issued have landed once the drain barrier flips.
      umma_commit(smem_u32(drain_bar));
      wait_drain(smem_u32(drain_bar), 0, kDrainBudget);
    }
  } else if (warp < kCombEpiWarp0) {
    // ------------------------------------------------- splitter warps
    const int row = threadIdx.x - kCombSplitWarp0 * 32;   // 0..127
    const int sw = row & 7;
    int c = 0;
    bool ok = true;
    for (int it = 0; it < rounds && ok; ++it) {
      Tile t;
      if (!tiles(it, t)) continue;
      for (int kb = 0; kb < num_kb; ++kb, ++c) {
        const int s = c % C::S;
        if (!(ok = wait_warp(smem_u32(full + s), (c / C::S) & 1, abort_flag, budget))) break;
        uint8_t* row_p = smem + s * C::STAGE + row * 128;   // c row, becomes the q+ row
        uint8_t* row_n = row_p + C::C_BYTES;                // q- row
        uint4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = *reinterpret_cast<const uint4*>(row_p + ((i ^ sw) << 4));
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          uint4 qp, qn;
          split4(v[i].x, qp.x, qn.x);
          split4(v[i].y, qp.y, qn.y);
          split4(v[i].z, qp.z, qn.z);
          split4(v[i].w, qp.w, qn.w);
          *reinterpret_cast<uint4*>(row_p + ((i ^ sw) << 4)) = qp;
          *reinterpret_cast<uint4*>(row_n + ((i ^ sw) << 4)) = qn;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(ready + s));
      }
    }
  } else {
    // --------------------------------------------------------- epilogue
    // Warp w reads TMEM lanes 32*(w % 4) .. +31; warps 6..(6+E-1) cover each
    // lane quarter once per column part.
    const int quad = warp & 3;
    const int part = (warp - kCombEpiWarp0) >> 2;
    epilogue_role<BN, C::NBUF, MULTI, false, Y_BF16, false>(
        args, quad, part, lane, tmem_base + ((uint32_t)(quad * 32) << 16), tmem_full,
        smem_u32(tmem_empty), /*empty_remote=*/false, /*row_shift=*/0, rounds, tiles, abort_flag,
        budget);
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_ALLOC);
  }
}

}  // namespace sq
