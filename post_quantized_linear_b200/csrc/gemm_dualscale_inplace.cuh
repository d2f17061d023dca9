// Fused DualScale GEMM with in-place activation quantization (bf16 X, int8 W).
//
// The same computation as dualscale_gemm_kernel with ASRC_X (SegQuant
// DualScale: X split by sign, each part quantized with its static scale, two
// int8 products per unit fused in the epilogue; see gemm_dualscale.cuh), with
// a different shared-memory plan.  A bf16 activation stage of 128 rows x 128 k
// is two 128-byte-swizzled boxes of 16 KiB; the two int8 operand tiles q+ and
// q- of the same k block are also 16 KiB each in the same swizzled layout.  The
// producer warps therefore quantize in place: q+ overwrites the first box and
// q- the second, and one ring of stages (activations, then codes, plus the
// weight tile) carries TMA -> quantizer -> MMA.  Without a separate code ring
// the pipeline holds twice as many k blocks in flight.
//
// Producer warps 2..9 form two groups of four that take alternate k blocks;
// in its group, thread t owns row t % 128 of the stage.  It reads the row's
// first box (k 0..63), writes those q+ codes over it and keeps the q- codes,
// then reads the second box (k 64..127), writes the remaining q+ codes into
// the first box and all q- codes over the second.  A box row is only
// overwritten by the thread that has already read it, so no barrier between
// threads is needed.
#pragma once

#include "gemm_dualscale.cuh"

namespace sq {

template <int BN_>
struct InplaceCfg {
  static constexpr int BN = BN_;
  static constexpr int A_BYTES = 2 * BM * 128;   // two bf16 boxes = q+ tile + q- tile
  static constexpr int W_BYTES = BN * BK;
  static constexpr int STAGE = A_BYTES + W_BYTES;
  static constexpr int S = (kStageBudget / STAGE) < 8 ? (kStageBudget / STAGE) : 8;
  static constexpr int NBUF = (BN <= 128) ? 2 : 1;
  static constexpr int OFF_BAR = S * STAGE;
  static constexpr int NUM_BARS = 3 * 8 + 2 * 2 + 1;  // full, ready, empty; tmem full/empty; drain
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int TMEM_COLS = 2 * BN * NBUF;
  static constexpr int TMEM_ALLOC = TMEM_COLS <= 256 ? 256 : 512;
  static_assert(S >= 2 && TMEM_COLS <= 512 && SMEM_BYTES <= 232448, "budgets");
};

template <int BN, bool ACC_OUT, bool Y_BF16, bool MULTI>
__global__ void __launch_bounds__(kernel_threads(MULTI), 1)
    dualscale_gemm_inplace_kernel(const __grid_constant__ CUtensorMap tmap_x,
                                  const __grid_constant__ CUtensorMap tmap_w,
                                  const __grid_constant__ GemmArgs args) {
  using C = InplaceCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;                  // [8] activations and weights landed
  uint64_t* ready = full + 8;             // [8] codes written in place
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
      mbar_init(smem_u32(ready + i), kProdWarps / 2);
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
      tma_prefetch_desc(&tmap_x);
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
          mbar_arrive_expect_tx(smem_u32(full + s), C::STAGE);
          tma_load_2d(smem_u32(st), &tmap_x, smem_u32(full + s), kb * BK, t.m0);
          tma_load_2d(smem_u32(st + BM * 128), &tmap_x, smem_u32(full + s), kb * BK + 64, t.m0);
          tma_load_2d(smem_u32(st + C::A_BYTES), &tmap_w, smem_u32(full + s), kb * BK, t.n0);
          ++c;
        }
      }
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
          const uint32_t a_n = a_p + BM * 128;
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
      umma_commit(smem_u32(drain_bar));
      wait_drain(smem_u32(drain_bar), 0, kDrainBudget);
    }
  } else if (warp < kEpiWarp0) {
    // ------------------------------------------ in-place quantizer warps
    const int t_id = threadIdx.x - kProdWarp0 * 32;  // 0..255
    const int row = t_id & (BM - 1);
    const int group = t_id >> 7;                     // takes k blocks with c % 2 == group
    const int sw = row & 7;
    int c = 0, cur_seg = -1;
    QuantParams qpar{0.0f, 0u, 0u};
    bool ok = true;
    for (int it = 0; it < rounds && ok; ++it) {
      Tile t;
      if (!tiles(it, t)) continue;
      for (int kb = 0; kb < num_kb; ++kb, ++c) {
        if ((c & 1) != group) continue;
        const int j = kb_segment(args, kb);
        if (j != cur_seg) {
          cur_seg = j;
          qpar = quant_params(__ldg(args.s_pos + j), __ldg(args.s_neg + j));
        }
        const int s = c % C::S;
        if (!(ok = wait_warp(smem_u32(full + s), (c / C::S) & 1, abort_flag, budget))) break;
        uint8_t* row_p = smem + s * C::STAGE + row * 128;  // box 0 row -> q+ row
        uint8_t* row_n = row_p + BM * 128;                 // box 1 row -> q- row
        uint4 qn_lo[4];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint8_t* src = half ? row_n : row_p;
          uint4 x[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) x[i] = *reinterpret_cast<const uint4*>(src + ((i ^ sw) << 4));
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            float v[16];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint32_t w[4] = {x[2 * g + h].x, x[2 * g + h].y, x[2 * g + h].z, x[2 * g + h].w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                v[8 * h + 2 * i] = __uint_as_float(w[i] << 16);
                v[8 * h + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
              }
            }
            uint4 qp, qn;
            quantize16_fast(v, qpar, qp, qn);
            *reinterpret_cast<uint4*>(row_p + (((half * 4 + g) ^ sw) << 4)) = qp;
            if (half == 0) {
              qn_lo[g] = qn;
            } else {
              *reinterpret_cast<uint4*>(row_n + (((4 + g) ^ sw) << 4)) = qn;
            }
          }
          if (half == 1) {
#pragma unroll
            for (int g = 0; g < 4; ++g)
              *reinterpret_cast<uint4*>(row_n + ((g ^ sw) << 4)) = qn_lo[g];
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(ready + s));
      }
    }
  } else {
    // --------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int part = (warp - kEpiWarp0) >> 2;
    epilogue_role<BN, C::NBUF, MULTI, ACC_OUT, Y_BF16, false>(
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
