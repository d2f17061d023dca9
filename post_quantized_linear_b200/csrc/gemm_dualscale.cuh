// Fused DualScale / SegLinear quantized linear for sm_100a.
//
// SegQuant ("SegQuant: A Semantics-Aware and Generalizable Quantization
// Framework for Diffusion Models"), Spanish technical summary 2.B and Korean
// technical summary section 2 "DualScale": X = X+ + X-, each part quantized
// with its own static scale; the products X+^ W^ and X-^ W^ run inside one
// kernel ("BatchedGEMM") and are combined in a fused epilogue.  Section 2.A /
// "SegLinear": every input segment carries its own activation and weight
// scales.
//
// The pages give no kernel; this one is designed for B200:
//   * warp 0      : TMA producer.  bf16/fp32 activation tiles (128 rows x 128 k,
//                   128-byte swizzle) and int8 weight tiles (BN rows x 128 k).
//   * warps 2..5  : quantizer.  Thread t owns tile row t: it reads its row of
//                   the activation stage, splits by sign, rounds half-to-even
//                   against each polarity's reciprocal scale and writes the two
//                   int8 operand tiles (q+ and q-) in the UMMA K-major 128-byte
//                   swizzled layout.
//   * warp 1      : TMEM allocator and the single MMA-issuing thread.  Per
//                   32-wide k step it issues two tcgen05.mma.kind::i8 (q+ W^T
//                   and q- W^T) sharing the weight descriptor, into two int32
//                   TMEM accumulators.  A unit (K segment, or 128-wide group
//                   for int4 weights) ends with a commit; accumulators are
//                   double-buffered across units (2 polarities x 2 buffers x BN
//                   columns = 512 TMEM columns for BN = 128).
//   * warps 6..13 : epilogue.  Per unit: tcgen05.ld of both accumulators,
//                   t = fmaf(s-, F(acc-), s+ * F(acc+)), y = fmaf(sw[n], t, y);
//                   after the last unit: + bias, convert, 16-byte stores.
// Every pipeline wait is bounded; on expiry the CTA records SQ_STATUS_TIMEOUT,
// lets in-flight copies and MMAs land, frees its TMEM and exits.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace sq {

constexpr int BM = 128;        // token rows per tile (UMMA M)
constexpr int BK = 128;        // k per pipeline stage (one 128-byte swizzle row of int8)
constexpr int kWarps = 14;
constexpr int kThreads = kWarps * 32;
constexpr int kQuantWarp0 = 2;  // warps 2..5
constexpr int kEpiWarp0 = 6;    // warps 6..13

struct GemmArgs {
  int32_t M, N, K;
  int32_t num_kb;          // ceil(K / BK)
  int32_t bits;            // 8 or 4
  SegBounds kseg;          // activation (and int8 weight) segments
  const float* s_pos;      // [J]
  const float* s_neg;      // [J]
  const void* wscales;     // fp32 [J][N] (bits 8) or binary16 [N][K/128] (bits 4)
  const float* bias;       // [N] or null
  void* y;                 // [M][ldy]
  int64_t ldy;
  int32_t* acc_out;        // [U][2][M][N] (accumulator mode)
  long long wait_budget;   // clock cycles per wait
};

template <int BN_, typename XT>
struct GemmCfg {
  static constexpr int BN = BN_;
  static constexpr int XE = (int)sizeof(XT);
  static constexpr int X_EPB = 128 / XE;                 // elements per 128-byte box row
  static constexpr int X_BOXES = BK / X_EPB;             // boxes per stage (2 bf16, 4 fp32)
  static constexpr int X_BOX_BYTES = BM * 128;
  static constexpr int X_STAGE = BM * BK * XE;
  static constexpr int W_STAGE = BN * BK;
  static constexpr int Q_TILE = BM * BK;
  static constexpr int Q_STAGE = 2 * Q_TILE;
  static constexpr int SX = 2;
  static constexpr int SW = (XE == 2) ? 4 : 2;
  static constexpr int SQ = (XE == 2) ? 3 : 2;
  static constexpr int OFF_X = 0;
  static constexpr int OFF_W = OFF_X + SX * X_STAGE;
  static constexpr int OFF_Q = OFF_W + SW * W_STAGE;
  static constexpr int OFF_BAR = OFF_Q + SQ * Q_STAGE;
  static constexpr int NUM_BARS = 2 * SX + 2 * SW + 2 * SQ + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  static constexpr int TMEM_COLS = 4 * BN;                 // 2 polarities x 2 buffers
  static_assert(TMEM_COLS <= 512, "TMEM holds 512 columns");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// --------------------------------------------------------------- waiting
// Single-thread bounded wait.  Returns false on timeout or when another role
// has already aborted.
__device__ __forceinline__ bool wait1(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                      long long budget) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > budget) {
      *abort_flag = 1;
      raise_status(SQ_STATUS_TIMEOUT);
      return false;
    }
  }
}

// Warp-uniform bounded wait: every lane observes the barrier itself (acquire),
// the loop exits together.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          long long budget) {
  const long long t0 = clock64();
  while (true) {
    const bool ok = mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, ok)) return true;
    int stop = 0;
    if ((threadIdx.x & 31) == 0) {
      if (*abort_flag) stop = 1;
      else if (clock64() - t0 > budget) {
        *abort_flag = 1;
        raise_status(SQ_STATUS_TIMEOUT);
        stop = 1;
      }
    }
    if (__shfl_sync(0xffffffffu, stop, 0)) return false;
  }
}

// Bounded wait used while tearing down: ignores the abort flag (the event
// waited for -- a bulk copy or an MMA landing -- completes on its own).
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity, long long budget) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > budget) {
      raise_status(SQ_STATUS_TIMEOUT);
      return;
    }
  }
}

// ----------------------------------------------------- quantizer helpers
// Reads 16 consecutive activations (k = 16c .. 16c+15) of tile row `row` from
// a 128-byte-swizzled activation stage.
template <typename XT>
__device__ __forceinline__ void load_row16(const uint8_t* xs, int row, int c, float (&v)[16]);

template <>
__device__ __forceinline__ void load_row16<__nv_bfloat16>(const uint8_t* xs, int row, int c,
                                                          float (&v)[16]) {
  const uint8_t* box = xs + (c >> 2) * (BM * 128) + row * 128;
  const int l0 = 2 * (c & 3);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint4 u = *reinterpret_cast<const uint4*>(box + (((l0 + h) ^ (row & 7)) << 4));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[8 * h + 2 * i] = __uint_as_float(w[i] << 16);
      v[8 * h + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

template <>
__device__ __forceinline__ void load_row16<float>(const uint8_t* xs, int row, int c,
                                                  float (&v)[16]) {
  const uint8_t* box = xs + (c >> 1) * (BM * 128) + row * 128;
  const int l0 = 4 * (c & 1);
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const float4 u = *reinterpret_cast<const float4*>(box + (((l0 + h) ^ (row & 7)) << 4));
    v[4 * h + 0] = u.x; v[4 * h + 1] = u.y; v[4 * h + 2] = u.z; v[4 * h + 3] = u.w;
  }
}

// Low bytes of four fp32 bit patterns, byte i from a_i.
__device__ __forceinline__ uint32_t low_bytes4(uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3) {
  return __byte_perm(__byte_perm(a0, a1, 0x0040), __byte_perm(a2, a3, 0x0040), 0x5410);
}

// DualScale rounding (see quant_kernels.cuh for the argument): the fma adds the
// exact product to 1.5*2^23, whose fp32 spacing is 1, so it rounds half to even
// to an integer; fmin/fmax clamp to [0,127] / [-127,0] in the float domain.
__device__ __forceinline__ void quantize16(const float (&v)[16], float rp, float rn, uint4& qp,
                                           uint4& qn) {
  uint32_t p[16], n[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    p[i] = __float_as_uint(fminf(fmaf(fmaxf(v[i], 0.0f), rp, kMagic), kMagic + 127.0f));
    n[i] = __float_as_uint(fmaxf(fmaf(fminf(v[i], 0.0f), rn, kMagic), kMagic - 127.0f));
  }
  qp.x = low_bytes4(p[0], p[1], p[2], p[3]);
  qp.y = low_bytes4(p[4], p[5], p[6], p[7]);
  qp.z = low_bytes4(p[8], p[9], p[10], p[11]);
  qp.w = low_bytes4(p[12], p[13], p[14], p[15]);
  qn.x = low_bytes4(n[0], n[1], n[2], n[3]);
  qn.y = low_bytes4(n[4], n[5], n[6], n[7]);
  qn.z = low_bytes4(n[8], n[9], n[10], n[11]);
  qn.w = low_bytes4(n[12], n[13], n[14], n[15]);
}

__device__ __forceinline__ float rcp_or_zero(float s) { return s > 0.0f ? __frcp_rn(s) : 0.0f; }

// Segment of the K block `kb` and whether it closes its unit.
__device__ __forceinline__ int kb_segment(const GemmArgs& a, int kb) {
  return a.kseg.segment_of(kb * BK);
}
__device__ __forceinline__ bool kb_closes_unit(const GemmArgs& a, int kb) {
  if (a.bits == 4 || kb + 1 == a.num_kb) return true;
  const int j = kb_segment(a, kb);
  return (kb + 1) * BK >= a.kseg.b[j + 1];
}

// ------------------------------------------------------------------ kernel
template <int BN, typename XT, bool ACC_OUT, bool Y_BF16>
__global__ void __launch_bounds__(kThreads, 1)
    dualscale_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x,
                          const __grid_constant__ CUtensorMap tmap_w,
                          const __grid_constant__ GemmArgs args) {
  using C = GemmCfg<BN, XT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sm_x = smem + C::OFF_X;
  uint8_t* sm_w = smem + C::OFF_W;
  uint8_t* sm_q = smem + C::OFF_Q;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full_x = bars;
  uint64_t* empty_x = full_x + C::SX;
  uint64_t* full_w = empty_x + C::SX;
  uint64_t* empty_w = full_w + C::SW;
  uint64_t* full_q = empty_w + C::SW;
  uint64_t* empty_q = full_q + C::SQ;
  uint64_t* tmem_full = empty_q + C::SQ;   // [2]
  uint64_t* tmem_empty = tmem_full + 2;    // [2]
  uint64_t* drain_bar = tmem_empty + 2;    // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * BM;
  const int n0 = blockIdx.x * BN;
  const long long budget = args.wait_budget;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::SX; ++i) { mbar_init(smem_u32(full_x + i), 1); mbar_init(smem_u32(empty_x + i), 4); }
    for (int i = 0; i < C::SW; ++i) { mbar_init(smem_u32(full_w + i), 1); mbar_init(smem_u32(empty_w + i), 1); }
    for (int i = 0; i < C::SQ; ++i) { mbar_init(smem_u32(full_q + i), 4); mbar_init(smem_u32(empty_q + i), 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(smem_u32(tmem_full + i), 1); mbar_init(smem_u32(tmem_empty + i), 8); }
    mbar_init(smem_u32(drain_bar), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_kb = args.num_kb;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_x);
      tma_prefetch_desc(&tmap_w);
      int issued_x = 0, issued_w = 0;
      for (int kb = 0; kb < num_kb; ++kb) {
        const int sx = issued_x % C::SX;
        const uint32_t px = (issued_x / C::SX) & 1;
        if (!wait1(smem_u32(empty_x + sx), px ^ 1, abort_flag, budget)) break;
        mbar_arrive_expect_tx(smem_u32(full_x + sx), C::X_STAGE);
        for (int b = 0; b < C::X_BOXES; ++b)
          tma_load_2d(smem_u32(sm_x + sx * C::X_STAGE + b * C::X_BOX_BYTES), &tmap_x,
                      smem_u32(full_x + sx), kb * BK + b * C::X_EPB, m0);
        ++issued_x;
        const int sw = issued_w % C::SW;
        const uint32_t pw = (issued_w / C::SW) & 1;
        if (!wait1(smem_u32(empty_w + sw), pw ^ 1, abort_flag, budget)) break;
        mbar_arrive_expect_tx(smem_u32(full_w + sw), C::W_STAGE);
        tma_load_2d(smem_u32(sm_w + sw * C::W_STAGE), &tmap_w, smem_u32(full_w + sw), kb * BK, n0);
        ++issued_w;
      }
      // Let every copy this thread started land before the CTA can exit.
      for (int s = 0; s < C::SX; ++s) {
        if (issued_x > s) {
          const int last = ((issued_x - 1 - s) / C::SX) * C::SX + s;
          wait_drain(smem_u32(full_x + s), (last / C::SX) & 1, budget);
        }
      }
      for (int s = 0; s < C::SW; ++s) {
        if (issued_w > s) {
          const int last = ((issued_w - 1 - s) / C::SW) * C::SW + s;
          wait_drain(smem_u32(full_w + s), (last / C::SW) & 1, budget);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(BM, BN);
      int unit = 0;
      bool unit_open = false;
      uint32_t d_pos = 0;
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!unit_open) {
          const int b = unit & 1;
          if (!wait1(smem_u32(tmem_empty + b), ((unit >> 1) & 1) ^ 1, abort_flag, budget)) break;
          tc_fence_after();
          d_pos = tmem_base + (uint32_t)(b * 2 * BN);
        }
        const int sw = kb % C::SW, sq = kb % C::SQ;
        if (!wait1(smem_u32(full_w + sw), (kb / C::SW) & 1, abort_flag, budget)) break;
        if (!wait1(smem_u32(full_q + sq), (kb / C::SQ) & 1, abort_flag, budget)) break;
        tc_fence_after();
        const uint32_t a_p = smem_u32(sm_q + sq * C::Q_STAGE);
        const uint32_t a_n = a_p + C::Q_TILE;
        const uint32_t b_w = smem_u32(sm_w + sw * C::W_STAGE);
#pragma unroll
        for (int ks = 0; ks < BK / 32; ++ks) {
          const uint32_t acc = (unit_open || ks > 0) ? 1u : 0u;
          const uint64_t bd = smem_desc_k_sw128(b_w + ks * 32);
          umma_i8(d_pos, smem_desc_k_sw128(a_p + ks * 32), bd, idesc, acc);
          umma_i8(d_pos + BN, smem_desc_k_sw128(a_n + ks * 32), bd, idesc, acc);
        }
        unit_open = true;
        umma_commit(smem_u32(empty_w + sw));
        umma_commit(smem_u32(empty_q + sq));
        if (kb_closes_unit(args, kb)) {
          umma_commit(smem_u32(tmem_full + (unit & 1)));
          ++unit;
          unit_open = false;
        }
      }
      // All MMAs this thread issued have landed once the drain barrier flips.
      umma_commit(smem_u32(drain_bar));
      wait_drain(smem_u32(drain_bar), 0, budget);
    }
  } else if (warp < kEpiWarp0) {
    // -------------------------------------------------------- quantizer
    const int row = threadIdx.x - kQuantWarp0 * 32;  // 0..127, tile row
    int cur_seg = -1;
    float rp = 0.0f, rn = 0.0f;
    for (int kb = 0; kb < num_kb; ++kb) {
      const int j = kb_segment(args, kb);
      if (j != cur_seg) {
        cur_seg = j;
        rp = rcp_or_zero(__ldg(args.s_pos + j));
        rn = rcp_or_zero(__ldg(args.s_neg + j));
      }
      const int sx = kb % C::SX, sq = kb % C::SQ;
      if (!wait_warp(smem_u32(full_x + sx), (kb / C::SX) & 1, abort_flag, budget)) break;
      if (!wait_warp(smem_u32(empty_q + sq), ((kb / C::SQ) & 1) ^ 1, abort_flag, budget)) break;
      const uint8_t* xs = sm_x + sx * C::X_STAGE;
      uint8_t* qp = sm_q + sq * C::Q_STAGE + row * 128;
      uint8_t* qn = qp + C::Q_TILE;
#pragma unroll 2
      for (int c = 0; c < 8; ++c) {
        float v[16];
        load_row16<XT>(xs, row, c, v);
        uint4 up, un;
        quantize16(v, rp, rn, up, un);
        const int off = (c ^ (row & 7)) << 4;
        *reinterpret_cast<uint4*>(qp + off) = up;
        *reinterpret_cast<uint4*>(qn + off) = un;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(empty_x + sx));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(full_q + sq));
    }
  } else {
    // --------------------------------------------------------- epilogue
    constexpr int HALF = BN / 2;
    const int quad = warp & 3;
    const int half = (warp - kEpiWarp0) >> 2;
    const int row = m0 + quad * 32 + lane;
    const int col0 = n0 + half * HALF;
    const uint32_t t_lane = tmem_base + ((uint32_t)(quad * 32) << 16);
    float y[HALF];
#pragma unroll
    for (int i = 0; i < HALF; ++i) y[i] = 0.0f;
    const int num_units = (args.bits == 4) ? num_kb : args.kseg.count;
    const int G = args.K / 128;
    bool ok = true;
    for (int u = 0; u < num_units; ++u) {
      const int b = u & 1;
      if (!wait_warp(smem_u32(tmem_full + b), (u >> 1) & 1, abort_flag, budget)) { ok = false; break; }
      tc_fence_after();
      const int j = (args.bits == 4) ? args.kseg.segment_of(u * 128) : u;
      const float sp = __ldg(args.s_pos + j), sn = __ldg(args.s_neg + j);
#pragma unroll
      for (int c = 0; c < HALF / 16; ++c) {
        uint32_t ap[16], an[16];
        const uint32_t col = (uint32_t)(b * 2 * BN + half * HALF + c * 16);
        tmem_ld16(t_lane + col, ap);
        tmem_ld16(t_lane + col + BN, an);
        tmem_wait_ld();
        const int n = col0 + c * 16;
        if constexpr (ACC_OUT) {
          if (row < args.M && n < args.N) {
            int32_t* dp = args.acc_out + (((int64_t)u * 2 + 0) * args.M + row) * args.N + n;
            int32_t* dn = args.acc_out + (((int64_t)u * 2 + 1) * args.M + row) * args.N + n;
#pragma unroll
            for (int i = 0; i < 16; i += 4) {
              *reinterpret_cast<uint4*>(dp + i) = make_uint4(ap[i], ap[i + 1], ap[i + 2], ap[i + 3]);
              *reinterpret_cast<uint4*>(dn + i) = make_uint4(an[i], an[i + 1], an[i + 2], an[i + 3]);
            }
          }
        } else {
          float sw[16];
          if (n < args.N) {
            if (args.bits == 8) {
              const float4* s4 = reinterpret_cast<const float4*>(
                  static_cast<const float*>(args.wscales) + (int64_t)j * args.N + n);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float4 t = __ldg(s4 + i);
                sw[4 * i] = t.x; sw[4 * i + 1] = t.y; sw[4 * i + 2] = t.z; sw[4 * i + 3] = t.w;
              }
            } else {
              const __half* hs = static_cast<const __half*>(args.wscales);
#pragma unroll
              for (int i = 0; i < 16; ++i) sw[i] = __half2float(hs[(int64_t)(n + i) * G + u]);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) sw[i] = 0.0f;
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float fp = __int2float_rn((int)ap[i]);
            const float fn = __int2float_rn((int)an[i]);
            const float t = __fmaf_rn(sn, fn, __fmul_rn(sp, fp));
            y[c * 16 + i] = __fmaf_rn(sw[i], t, y[c * 16 + i]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(tmem_empty + b));
    }
    if constexpr (!ACC_OUT) {
      if (ok && row < args.M) {
#pragma unroll
        for (int c = 0; c < HALF / 16; ++c) {
          const int n = col0 + c * 16;
          if (n < args.N) {
            float o[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = y[c * 16 + i];
            if (args.bias != nullptr) {
              const float4* b4 = reinterpret_cast<const float4*>(args.bias + n);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float4 t = __ldg(b4 + i);
                o[4 * i] = __fadd_rn(o[4 * i], t.x);
                o[4 * i + 1] = __fadd_rn(o[4 * i + 1], t.y);
                o[4 * i + 2] = __fadd_rn(o[4 * i + 2], t.z);
                o[4 * i + 3] = __fadd_rn(o[4 * i + 3], t.w);
              }
            }
            if constexpr (Y_BF16) {
              __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(args.y) + (int64_t)row * args.ldy + n;
              uint32_t pk[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(o[2 * i], o[2 * i + 1]);
                pk[i] = *reinterpret_cast<const uint32_t*>(&h2);
              }
              reinterpret_cast<uint4*>(dst)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              reinterpret_cast<uint4*>(dst)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            } else {
              float* dst = static_cast<float*>(args.y) + (int64_t)row * args.ldy + n;
#pragma unroll
              for (int i = 0; i < 4; ++i)
                reinterpret_cast<float4*>(dst)[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
            }
          }
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace sq
