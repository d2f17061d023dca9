// DualScale GEMM from codes for small M (M <= 128): split-K over the whole GPU.
//
// With one row tile the work is streaming the weight codes (N x K bytes) from
// HBM; one CTA per N tile would leave most SMs idle.  Each (N tile, K split)
// pair is a unit: the unit's CTA runs the two int8 products (SegQuant
// DualScale, section "DualScale" of the SegQuant paper) over its K range into
// TMEM, and every epilogue warp writes its part of the int32 partial
// accumulators to a workspace.  Integer partial sums add exactly, in any
// order, so the result is bit-identical to the one-pass kernels.
//
// Reduction without waiting: a warp publishes its partial (stores,
// __threadfence) and then increments the counter of its (tile, warp region);
// the warp that sees the count reach `splits - 1` is the last, and it alone
// adds the other splits' partials (read past L1) to its own accumulators,
// still in TMEM, folds them and writes Y, then resets the counter to 0 for the
// next call.  No CTA ever waits for another.  The workspace's counters must be
// zero before the first call; a completed call leaves them zero.
//
// Pipeline per CTA: warp 0 TMA (q+, q-, weight tile per k block, one ring),
// warp 1 TMEM + MMA, warps 2..9 epilogue -- the layout of the one-ring codes
// kernel (gemm_dualscale_codes.cuh).
#pragma once

#include "gemm_dualscale.cuh"
#include "gemm_dualscale_codes.cuh"

namespace sq {

template <int BN_>
struct SplitKCfg {
  static constexpr int BN = BN_;
  static constexpr int A_BYTES = 2 * BM * BK;
  static constexpr int W_BYTES = BN * BK;
  static constexpr int STAGE = A_BYTES + W_BYTES;
  static constexpr int S = (kStageBudget / STAGE) < 8 ? (kStageBudget / STAGE) : 8;
  static constexpr int NBUF = (4 * BN <= 512) ? 2 : 1;
  static constexpr int OFF_BAR = S * STAGE;
  static constexpr int NUM_BARS = 2 * 8 + 2 * 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int TMEM_COLS = 2 * BN * NBUF;
  static constexpr int TMEM_ALLOC = TMEM_COLS <= 256 ? 256 : 512;
  static constexpr int EPW = 8;                      // epilogue warps = counter regions per tile
  static constexpr int HALF = BN / (EPW / 4);        // columns per epilogue warp
  static_assert(S >= 2 && TMEM_COLS <= 512 && SMEM_BYTES <= 232448, "budgets");
  static_assert(HALF % 16 == 0, "16-column chunks");
};

// The unit handled in round `it` by this CTA: tile (N index), K split, k-block range.
struct SplitUnit {
  int tile, split, kb0, kb1, n0, width;
};

__device__ __forceinline__ bool split_unit_of(const GemmArgs& a, int bn, int it, SplitUnit& u) {
  const int idx = it * (int)gridDim.x + (int)blockIdx.x;
  if (idx >= a.num_tiles * a.splits) return false;
  u.tile = idx / a.splits;
  u.split = idx - u.tile * a.splits;
  u.kb0 = u.split * a.kb_per_split;
  u.kb1 = min(u.kb0 + a.kb_per_split, a.num_kb);
  u.n0 = u.tile * bn;
  u.width = min(bn, a.N - u.n0);
  return true;
}

template <int BN, bool Y_BF16>
__global__ void __launch_bounds__(codes_kernel_threads(false), 1)
    dualscale_gemm_splitk_kernel(const __grid_constant__ CUtensorMap tmap_qp,
                                 const __grid_constant__ CUtensorMap tmap_qn,
                                 const __grid_constant__ CUtensorMap tmap_w,
                                 const __grid_constant__ GemmArgs args) {
  using C = SplitKCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;                  // [8]
  uint64_t* empty = full + 8;             // [8]
  uint64_t* tmem_full = empty + 8;        // [2]
  uint64_t* tmem_empty = tmem_full + 2;   // [2]
  uint64_t* drain_bar = tmem_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long budget = args.wait_budget;
  const int rounds = (args.num_tiles * args.splits + (int)gridDim.x - 1) / (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::S; ++i) {
      mbar_init(smem_u32(full + i), 1);
      mbar_init(smem_u32(empty + i), 1);
    }
    for (int i = 0; i < C::NBUF; ++i) {
      mbar_init(smem_u32(tmem_full + i), 1);
      mbar_init(smem_u32(tmem_empty + i), C::EPW);
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

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_qp);
      tma_prefetch_desc(&tmap_qn);
      tma_prefetch_desc(&tmap_w);
      int c = 0;
      bool ok = (args.starve == 0);
      for (int it = 0; it < rounds && ok; ++it) {
        SplitUnit u;
        if (!split_unit_of(args, BN, it, u)) break;
        for (int kb = u.kb0; kb < u.kb1; ++kb) {
          const int s = c % C::S;
          if (!(ok = wait1(smem_u32(empty + s), ((c / C::S) & 1) ^ 1, abort_flag, budget))) break;
          uint8_t* st = smem + s * C::STAGE;
          mbar_arrive_expect_tx(smem_u32(full + s), C::STAGE);
          tma_load_2d(smem_u32(st), &tmap_qp, smem_u32(full + s), kb * BK, 0);
          tma_load_2d(smem_u32(st + BM * BK), &tmap_qn, smem_u32(full + s), kb * BK, 0);
          tma_load_2d(smem_u32(st + C::A_BYTES), &tmap_w, smem_u32(full + s), kb * BK, u.n0);
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
        SplitUnit u;
        if (!split_unit_of(args, BN, it, u)) break;
        const uint32_t idesc = idesc_i8(BM, u.width);
        const int b = ug % C::NBUF;
        if (!(ok = wait1(smem_u32(tmem_empty + b), ((ug / C::NBUF) & 1) ^ 1, abort_flag, budget))) break;
        tc_fence_after();
        const uint32_t d_pos = tmem_base + (uint32_t)(b * 2 * BN);
        for (int kb = u.kb0; kb < u.kb1; ++kb) {
          const int s = c % C::S;
          if (!(ok = wait1(smem_u32(full + s), (c / C::S) & 1, abort_flag, budget))) break;
          const uint32_t a_p = smem_u32(smem + s * C::STAGE);
          const uint32_t a_n = a_p + BM * BK;
          const uint32_t b_w = a_p + C::A_BYTES;
#pragma unroll
          for (int ks = 0; ks < BK / 32; ++ks) {
            const uint32_t acc = (kb > u.kb0 || ks > 0) ? 1u : 0u;
            const uint64_t bd = smem_desc_k_sw128(b_w + ks * 32);
            umma_i8(d_pos, smem_desc_k_sw128(a_p + ks * 32), bd, idesc, acc);
            umma_i8(d_pos + BN, smem_desc_k_sw128(a_n + ks * 32), bd, idesc, acc);
          }
          umma_commit(smem_u32(empty + s));
          ++c;
        }
        if (!ok) break;
        umma_commit(smem_u32(tmem_full + b));
        ++ug;
      }
      umma_commit(smem_u32(drain_bar));
      wait_drain(smem_u32(drain_bar), 0, kDrainBudget);
    }
  } else {
    // --------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int part = (warp - kCodesEpiWarp0) >> 2;
    const int region = warp - kCodesEpiWarp0;          // 0..7: counter index within a tile
    const uint32_t t_lane = tmem_base + ((uint32_t)(quad * 32) << 16);
    const int row = quad * 32 + lane;                  // tile row = output row (one row tile)
    const int64_t slice = (int64_t)args.M * args.N;    // int32 elements of one (split, polarity)
    const float sp = __ldg(args.s_pos), sn = __ldg(args.s_neg);
    int ug = 0;
    bool ok = true;
    for (int it = 0; it < rounds && ok; ++it) {
      SplitUnit u;
      if (!split_unit_of(args, BN, it, u)) break;
      const int b = ug % C::NBUF;
      if (!(ok = wait_warp(smem_u32(tmem_full + b), (ug / C::NBUF) & 1, abort_flag, budget))) break;
      tc_fence_after();
      const int c_lo = part * C::HALF;
      const int cols = min(C::HALF, u.width - c_lo);
      if (quad * 32 < args.M && cols > 0) {
        // 1. publish this split's partial accumulators (rows < M)
        int32_t* mine = args.ws_part + (int64_t)(u.split * 2) * slice;
        for (int c = 0; c < cols; c += 16) {
          uint32_t ap[16], an[16];
          const uint32_t col = (uint32_t)(b * 2 * BN + c_lo + c);
          tmem_ld16(t_lane + col, ap);
          tmem_ld16(t_lane + col + BN, an);
          tmem_wait_ld();
          if (row < args.M) {
            uint4* dp = reinterpret_cast<uint4*>(mine + (int64_t)row * args.N + u.n0 + c_lo + c);
            uint4* dn = reinterpret_cast<uint4*>(mine + slice + (int64_t)row * args.N + u.n0 + c_lo + c);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              dp[i] = make_uint4(ap[4 * i], ap[4 * i + 1], ap[4 * i + 2], ap[4 * i + 3]);
              dn[i] = make_uint4(an[4 * i], an[4 * i + 1], an[4 * i + 2], an[4 * i + 3]);
            }
          }
        }
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) {
          const int old = atomicAdd(args.ws_count + u.tile * C::EPW + region, 1);
          last = (old == args.splits - 1);
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
          // 2. the last split: sum every split's partial, fold, store Y
          __threadfence();
          for (int c = 0; c < cols; c += 16) {
            uint32_t ap[16], an[16];
            const uint32_t col = (uint32_t)(b * 2 * BN + c_lo + c);
            tmem_ld16(t_lane + col, ap);
            tmem_ld16(t_lane + col + BN, an);
            tmem_wait_ld();
            if (row < args.M) {
              const int n = u.n0 + c_lo + c;
              for (int s2 = 0; s2 < args.splits; ++s2) {
                if (s2 == u.split) continue;
                const int32_t* src = args.ws_part + (int64_t)(s2 * 2) * slice + (int64_t)row * args.N + n;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const int4 vp = __ldcg(reinterpret_cast<const int4*>(src) + i);
                  const int4 vn = __ldcg(reinterpret_cast<const int4*>(src + slice) + i);
                  ap[4 * i] += (uint32_t)vp.x; ap[4 * i + 1] += (uint32_t)vp.y;
                  ap[4 * i + 2] += (uint32_t)vp.z; ap[4 * i + 3] += (uint32_t)vp.w;
                  an[4 * i] += (uint32_t)vn.x; an[4 * i + 1] += (uint32_t)vn.y;
                  an[4 * i + 2] += (uint32_t)vn.z; an[4 * i + 3] += (uint32_t)vn.w;
                }
              }
              float sw[16], o[16];
              load_wscales16(args, 0, 0, n, sw);
#pragma unroll
              for (int i = 0; i < 16; ++i) o[i] = 0.0f;
              fold16<false>(ap, an, sw, sp, sn, o);
              store16<Y_BF16>(args, row, n, o);
            }
          }
          if (lane == 0) args.ws_count[u.tile * C::EPW + region] = 0;   // ready for the next call
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(tmem_empty + b));
      ++ug;
    }
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
