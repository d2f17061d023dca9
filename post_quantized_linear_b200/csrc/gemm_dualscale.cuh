// Fused DualScale / SegLinear quantized linear for sm_100a (W8A8 and W4A8).
//
// SegQuant ("SegQuant: A Semantics-Aware and Generalizable Quantization
// Framework for Diffusion Models"), Spanish technical summary 2.B and Korean
// technical summary section 2 "DualScale": X = X+ + X-, each part quantized
// with its own static scale; the products X+^ W^ and X-^ W^ run inside one
// kernel ("BatchedGEMM") and are combined in a fused epilogue.  Section 2.A /
// "SegLinear": every input segment carries its own activation and weight
// scales.  W4A8 (Spanish technical summary 4, results): 4-bit weights.
//
// The pages give no kernel; this one is designed for B200.  Persistent: one
// CTA per SM walks output tiles (128 rows x BN columns) in a snake order, and
// every ring below runs continuously across tiles.
//   * warp 0       : TMA producer.  Activation tiles (128 rows x 128 k,
//                    128-byte swizzle) or, for pre-quantized activations, the
//                    two int8 code tiles; int8 weight tiles (BN x 128 k) or
//                    packed int4 weight tiles (BN x 64 bytes).
//   * warps 2..9   : operand producers.  Fused mode: thread t owns tile row
//                    t % 128 and half of its k range; it splits each activation
//                    by sign, rounds half-to-even against each polarity's
//                    reciprocal scale and writes q+ and q- in the UMMA K-major
//                    128-byte swizzled layout.  int4 weights: the packed tile
//                    is sign-extended to int8 in the same layout.
//   * warp 1       : TMEM allocator and the single MMA-issuing thread.  Per
//                    32-wide k step, two tcgen05.mma.kind::i8 (q+ W^T, q- W^T)
//                    share the weight descriptor and accumulate into two int32
//                    TMEM accumulators.  A unit (K segment, or 128-wide group
//                    for int4 weights) ends with a commit; with BN = 128 the
//                    accumulators are double-buffered (2 x 2 x 128 = 512 TMEM
//                    columns), so the epilogue of one unit or tile overlaps the
//                    MMAs of the next.
//   * warps 10..17 : epilogue.  tcgen05.ld of both accumulators;
//                    t = fmaf(s-, F(acc-), s+ * F(acc+)), y = fmaf(sw[n], t, y);
//                    after the last unit: + bias, convert, 16-byte stores.
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

constexpr int BM = 128;  // token rows per tile (UMMA M)
constexpr int BK = 128;  // k per pipeline stage (one 128-byte swizzle row of int8)
constexpr int kProdWarp0 = 2;
constexpr int kProdWarps = 8;
constexpr int kEpiWarp0 = kProdWarp0 + kProdWarps;  // 10

// Epilogue warps: 8 for one unit per tile (columns streamed from TMEM), 16
// when partial outputs must stay in registers across units (32 columns per
// thread).  Registers are granted in 4-warp groups, so 18 warps get at most
// 96 registers per thread and 26 warps 72.
__host__ __device__ constexpr int epi_warps(bool multi) { return multi ? 16 : 8; }
__host__ __device__ constexpr int kernel_threads(bool multi) {
  return (kEpiWarp0 + epi_warps(multi)) * 32;
}

// Source of the A operand.
constexpr int ASRC_X = 0;      // activations, quantized inside the kernel
constexpr int ASRC_CODES = 1;  // pre-quantized q+ / q- code tensors

struct GemmArgs {
  int32_t M, N, K;
  int32_t num_kb;          // ceil(K / BK)
  int32_t bits;            // 8 or 4
  int32_t n_full;          // number of full-width N tiles
  int32_t tail;            // width of the last, narrower N tile (0: none)
  int32_t m_tiles;         // ceil(M / BM)
  int32_t num_tiles;
  SegBounds kseg;          // activation (and int8 weight) segments
  const float* s_pos;      // [J]
  const float* s_neg;      // [J]
  const void* wscales;     // fp32 [J][N] (bits 8) or binary16 [K/128][N] (bits 4)
  const float* bias;       // [N] or null
  void* y;                 // [M][ldy]
  int64_t ldy;
  int32_t* acc_out;        // [U][2][M][N] (accumulator mode)
  long long wait_budget;   // clock cycles per pipeline wait
  int32_t starve;          // test hook: the TMA producer issues nothing
  // split-K (small M): K splits per N tile, k blocks per split, workspace
  int32_t splits;
  int32_t kb_per_split;
  int32_t* ws_count;       // [num_tiles][8] arrival counters (zero between calls)
  int32_t* ws_part;        // [splits][2][M][N] partial accumulators
  // activation codes read by cp.async loader warps (GEMM from codes)
  const int8_t* a_pos;     // q+ (or the single code) [M][lda]
  const int8_t* a_neg;     // q- [M][lda]
  int64_t lda;
  // Rows of one code-tile TMA box (GEMM from codes): BM, or M rounded up to 16
  // when a single row tile holds fewer than BM rows (0 means BM).  The rows
  // past the box keep stale shared memory; their accumulator lanes are never
  // stored.
  int32_t a_rows;
  // Stacked rows: tmap_qp is a 4-D map (K bytes x 16 rows x {q+, q-} x groups
  // of 16 rows) whose one box per k block lands every whole group's q+ and q-
  // rows in the stacked order (1); when M is not whole groups, tmap_qn is a
  // 3-D map (K bytes x M rows x {q+, q-}) that brings the last, partial group
  // in two 16-row boxes (2); or each group and polarity comes as its own
  // 16-row box of the 2-D maps (0).
  int32_t code_box4;
  int32_t code_neg_first;   // (code_box4) the map starts at q-: each group's q- rows come first
};

// Teardown waits (copies and MMAs that were issued always complete) get a
// fixed budget of about two seconds, independent of the pipeline-wait budget.
constexpr long long kDrainBudget = 4000000000LL;

constexpr int kStageBudget = 229376;  // 224 KiB of pipeline stages

template <int BN_, int ASRC_, typename XT, bool W4_>
struct GemmCfg {
  static constexpr int BN = BN_;
  static constexpr int ASRC = ASRC_;
  static constexpr bool W4 = W4_;
  static constexpr int XE = (int)sizeof(XT);
  static constexpr int X_EPB = 128 / XE;                 // elements per 128-byte box row
  static constexpr int X_BOXES = BK / X_EPB;             // boxes per stage (2 bf16, 4 fp32)
  static constexpr int X_BOX_BYTES = BM * 128;
  static constexpr int X_STAGE = (ASRC == ASRC_X) ? BM * BK * XE : 0;
  static constexpr int WP_STAGE = W4 ? BN * (BK / 2) : 0;  // packed int4 rows of 64 bytes
  static constexpr int W_STAGE = BN * BK;
  static constexpr int Q_TILE = BM * BK;
  static constexpr int Q_STAGE = 2 * Q_TILE;
  static constexpr bool BIG_X = (ASRC == ASRC_X) && XE == 4;
  static constexpr int SX = (ASRC == ASRC_X) ? 2 : 0;
  static constexpr int SWP = W4 ? (BIG_X ? 2 : 4) : 0;
  static constexpr int SW = W4 ? (BIG_X ? 1 : (ASRC == ASRC_CODES ? 3 : 2))
                               : (ASRC == ASRC_CODES ? (BN == 128 ? 4 : 3) : ((BIG_X || BN >= 192) ? 2 : 4));
  static constexpr int SQ = (kStageBudget - SX * X_STAGE - SWP * WP_STAGE - SW * W_STAGE) / Q_STAGE;
  static constexpr int NBUF = (BN <= 128) ? 2 : 1;       // TMEM accumulator buffers
  static constexpr int OFF_X = 0;
  static constexpr int OFF_WP = OFF_X + SX * X_STAGE;
  static constexpr int OFF_W = OFF_WP + SWP * WP_STAGE;
  static constexpr int OFF_Q = OFF_W + SW * W_STAGE;
  static constexpr int OFF_BAR = OFF_Q + SQ * Q_STAGE;
  static constexpr int NUM_BARS = 2 * 2 + 2 * 4 + 2 * 4 + 2 * 8 + 2 * 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  static constexpr int TMEM_COLS = 2 * BN * NBUF;
  static constexpr int TMEM_ALLOC = TMEM_COLS <= 256 ? 256 : 512;  // a power of two
  static_assert(TMEM_COLS <= 512, "TMEM holds 512 columns");
  static_assert(BN % 16 == 0 && BN <= 256, "UMMA N for M = 128");
  static_assert(SQ >= 2 && SQ <= 8 && SW >= 1 && SW <= 4 && SWP <= 4, "stage counts");
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

// Phase test with acquire at CTA scope, or at cluster scope for barriers that
// receive arrivals from the other CTA of a pair.
template <bool CLUSTER>
__device__ __forceinline__ bool try_wait_scoped(uint32_t bar, uint32_t parity) {
  if constexpr (CLUSTER) return mbar_try_wait_cluster(bar, parity);
  else return mbar_try_wait(bar, parity);
}

// Single-thread bounded wait with a selectable acquire scope.
template <bool CLUSTER>
__device__ __forceinline__ bool wait1s(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                       long long budget) {
  if (try_wait_scoped<CLUSTER>(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (try_wait_scoped<CLUSTER>(bar, parity)) return true;
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
template <bool CLUSTER = false>
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          long long budget) {
  if (__all_sync(0xffffffffu, try_wait_scoped<CLUSTER>(bar, parity))) return true;
  const long long t0 = clock64();
  while (true) {
    // a waiting warp sleeps between polls instead of taking issue slots from
    // the warps that are computing
    __nanosleep(64);
    const bool ok = try_wait_scoped<CLUSTER>(bar, parity);
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

// Waits for the last completion of every stage of a ring that `issued` loads
// were armed on (stage i % S, phase i / S).
__device__ __forceinline__ void drain_ring(const uint64_t* full, int S, int issued,
                                           long long budget) {
  for (int s = 0; s < S; ++s) {
    if (issued > s) {
      const int last = ((issued - 1 - s) / S) * S + s;
      wait_drain(smem_u32(full + s), (last / S) & 1, budget);
    }
  }
}

// ---------------------------------------------------------- tile schedule
struct Tile {
  int m0, n0, width;
};

// Tiles: full-width tiles first (row-major over (m, n)), then the narrower
// last-column tiles.  Round `it` of CTA `cta` takes tile it*ncta + pos, with
// pos reversed on odd rounds (snake) so that CTAs that drew short tiles in one
// round draw long ones in the next.
__device__ __forceinline__ bool tile_of(const GemmArgs& a, int it, int bn, Tile& t) {
  const int ncta = gridDim.x;
  const int pos = (it & 1) ? (ncta - 1 - (int)blockIdx.x) : (int)blockIdx.x;
  const int idx = it * ncta + pos;
  if (idx >= a.num_tiles) return false;
  const int nfull_tiles = a.m_tiles * a.n_full;
  if (idx < nfull_tiles) {
    t.m0 = (idx / a.n_full) * BM;
    t.n0 = (idx % a.n_full) * bn;
    t.width = bn;
  } else {
    t.m0 = (idx - nfull_tiles) * BM;
    t.n0 = a.n_full * bn;
    t.width = a.tail;
  }
  return true;
}

__device__ __forceinline__ int num_rounds(const GemmArgs& a) {
  return (a.num_tiles + gridDim.x - 1) / gridDim.x;
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

// Eight int4 codes (two per byte, low nibble = even k) -> eight int8 codes.
// A nibble n in 0..15 sign-extends to n | 0xF0 when bit 3 is set: the bit,
// multiplied by 30 (8 * 30 = 0xF0), lands in the high nibble of its own byte.
__device__ __forceinline__ uint2 unpack8_int4(uint32_t w) {
  uint32_t lo = w & 0x0F0F0F0Fu;
  uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;
  lo |= (lo & 0x08080808u) * 30u;
  hi |= (hi & 0x08080808u) * 30u;
  return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}

// Eight int4 codes (two per byte, low nibble = even k) -> eight int8 bytes
// holding 16 x the code: each nibble moved to the high half of its byte, whose
// sign bit it then carries (used with the 1.5 * 2^19 accumulator seed).
__device__ __forceinline__ uint2 unpack8_int4_x16(uint32_t w) {
  const uint32_t even = (w << 4) & 0xF0F0F0F0u;
  const uint32_t odd = w & 0xF0F0F0F0u;
  return make_uint2(__byte_perm(even, odd, 0x5140), __byte_perm(even, odd, 0x7362));
}

__device__ __forceinline__ float rcp_or_zero(float s) { return s > 0.0f ? __frcp_rn(s) : 0.0f; }

// Per-segment constants of the fused quantizer.
struct QuantParams {
  float lo;       // inputs below lo behave as lo: the -127 clamp, applied on the input
  uint32_t rp;    // bit pattern of r+ = 1/s+
  uint32_t dr;    // r- bits minus r+ bits (mod 2^32): rp + sign * dr selects r-
};

// The smallest fp32 L with L * r- > -127.5 (exact real product).  Every
// x >= L rounds to a code >= -127 and every x < L to one <= -128, which the
// clamp turns into -127 = rne(L * r-); so clamping x at L first is exact.
// fmaf(L, r, 127.5) rounds L*r + 127.5 once, and rounding keeps the sign, so
// each test below is exact.
__device__ __forceinline__ float neg_input_limit(float rn) {
  if (!(rn > 0.0f)) return -__int_as_float(0x7f800000);  // no negative branch: all codes 0
  float L = -127.5f / rn;
  for (int i = 0; i < 4 && !(fmaf(L, rn, 127.5f) > 0.0f); ++i) L = nextafterf(L, 0.0f);
  for (int i = 0; i < 4; ++i) {
    const float d = nextafterf(L, -__int_as_float(0x7f800000));
    if (fmaf(d, rn, 127.5f) > 0.0f) L = d;
    else break;
  }
  return L;
}

__device__ __forceinline__ QuantParams quant_params(float sp, float sn) {
  const float rp = rcp_or_zero(sp), rn = rcp_or_zero(sn);
  QuantParams q;
  q.lo = neg_input_limit(rn);
  q.rp = __float_as_uint(rp);
  q.dr = __float_as_uint(rn) - q.rp;
  return q;
}

// One DualScale code for an input already clamped below at QuantParams::lo:
// the sign bit (IMAD.HI) selects r- or r+ (IMAD), the fma rounds the exact
// product half-to-even against 1.5*2^23, and the bit difference is the signed
// code (large positive values saturate in the pack below).
__device__ __forceinline__ int32_t signed_code(float xc, const QuantParams& p) {
  const uint32_t sgn = __umulhi(__float_as_uint(xc), 2u);
  const float r = __uint_as_float(p.rp + sgn * p.dr);
  return (int32_t)(__float_as_uint(fmaf(xc, r, kMagic)) - kMagicBits);
}

// Four signed codes -> four bytes, each saturated to [-128, 127]; byte i from c_i.
__device__ __forceinline__ uint32_t pack_sat4(int32_t c0, int32_t c1, int32_t c2, int32_t c3) {
  uint32_t hi, out;
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, 0;" : "=r"(hi) : "r"(c3), "r"(c2));
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(out) : "r"(c1), "r"(c0), "r"(hi));
  return out;
}

// Splits four signed codes into their non-negative and negative parts (the
// other part's byte is 0): a byte's sign, replicated, selects it.
__device__ __forceinline__ void split4(uint32_t c, uint32_t& qp, uint32_t& qn) {
  uint32_t m;  // prmt with selector nibbles 8..11: each byte's sign bit, replicated
  asm("prmt.b32 %0, %1, 0, 0xBA98;" : "=r"(m) : "r"(c));
  qp = c & ~m;
  qn = c & m;
}

// 16 activations of one row -> 16 q+ and 16 q- codes.
__device__ __forceinline__ void quantize16_fast(const float (&v)[16], const QuantParams& p,
                                                uint4& qp, uint4& qn) {
  uint32_t w[4];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    int32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = signed_code(fmaxf(v[4 * g + i], p.lo), p);
    w[g] = pack_sat4(c[0], c[1], c[2], c[3]);
  }
  split4(w[0], qp.x, qn.x);
  split4(w[1], qp.y, qn.y);
  split4(w[2], qp.z, qn.z);
  split4(w[3], qp.w, qn.w);
}

// Segment of the K block `kb` and whether it closes its unit.
__device__ __forceinline__ int kb_segment(const GemmArgs& a, int kb) {
  return a.kseg.segment_of(kb * BK);
}
__device__ __forceinline__ bool kb_closes_unit(const GemmArgs& a, int kb) {
  if (a.bits == 4 || kb + 1 == a.num_kb) return true;
  const int j = kb_segment(a, kb);
  return (kb + 1) * BK >= a.kseg.b[j + 1];
}

// ------------------------------------------------------------- epilogue
// Weight scales of 16 consecutive output channels for unit u.
__device__ __forceinline__ void load_wscales16(const GemmArgs& a, int u, int j, int n,
                                               float (&sw)[16]) {
  if (a.bits == 8) {
    const float4* s4 =
        reinterpret_cast<const float4*>(static_cast<const float*>(a.wscales) + (int64_t)j * a.N + n);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 t = __ldg(s4 + i);
      sw[4 * i] = t.x; sw[4 * i + 1] = t.y; sw[4 * i + 2] = t.z; sw[4 * i + 3] = t.w;
    }
  } else {
    const uint4* h8 = reinterpret_cast<const uint4*>(static_cast<const __half*>(a.wscales) +
                                                     (int64_t)u * a.N + n);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint4 t = __ldg(h8 + i);
      const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
        sw[8 * i + 2 * k] = f.x;
        sw[8 * i + 2 * k + 1] = f.y;
      }
    }
  }
}

// int32 -> fp32, round to nearest even.  With |v| < 2^22 (int4 units) the
// magic-number form is exact: the pattern 0x4B400000 + v is the float
// 1.5*2^23 + v, and the subtraction is exact.
template <bool SMALL>
__device__ __forceinline__ float acc_to_f32(uint32_t v) {
  if constexpr (SMALL) return __uint_as_float(v + kMagicBits) - kMagic;
  else return __int2float_rn((int)v);
}

// y (+)= sw * (s- F(acc-) + s+ F(acc+)) in the fixed fp32 order.
template <bool SMALL>
__device__ __forceinline__ void fold16(const uint32_t (&ap)[16], const uint32_t (&an)[16],
                                       const float (&sw)[16], float sp, float sn, float* y) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float fp = acc_to_f32<SMALL>(ap[i]);
    const float fn = acc_to_f32<SMALL>(an[i]);
    const float t = __fmaf_rn(sn, fn, __fmul_rn(sp, fp));
    y[i] = __fmaf_rn(sw[i], t, y[i]);
  }
}

__device__ __forceinline__ void load_wscales8(const GemmArgs& a, int u, int j, int n,
                                              float (&sw)[8]) {
  if (a.bits == 8) {
    const float4* s4 =
        reinterpret_cast<const float4*>(static_cast<const float*>(a.wscales) + (int64_t)j * a.N + n);
    const float4 t0 = __ldg(s4), t1 = __ldg(s4 + 1);
    sw[0] = t0.x; sw[1] = t0.y; sw[2] = t0.z; sw[3] = t0.w;
    sw[4] = t1.x; sw[5] = t1.y; sw[6] = t1.z; sw[7] = t1.w;
  } else {
    const uint4 t = __ldg(reinterpret_cast<const uint4*>(static_cast<const __half*>(a.wscales) +
                                                         (int64_t)u * a.N + n));
    const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
      sw[2 * k] = f.x;
      sw[2 * k + 1] = f.y;
    }
  }
}

template <bool SMALL>
__device__ __forceinline__ void fold8(const uint32_t (&ap)[8], const uint32_t (&an)[8],
                                      const float (&sw)[8], float sp, float sn, float* y) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float fp = acc_to_f32<SMALL>(ap[i]);
    const float fn = acc_to_f32<SMALL>(an[i]);
    const float t = __fmaf_rn(sn, fn, __fmul_rn(sp, fp));
    y[i] = __fmaf_rn(sw[i], t, y[i]);
  }
}

// Prefetches into L1 the weight scales this thread will read for unit u:
// `cols` consecutive columns from tile column n (fp32 [J][N] or fp16 [G][N]).
__device__ __forceinline__ void prefetch_wscales(const GemmArgs& a, int u, int j, int n, int cols) {
  if (a.bits == 8) {
    const float* p = static_cast<const float*>(a.wscales) + (int64_t)j * a.N + n;
    for (int c = 0; c < cols; c += 32) prefetch_l1(p + c);
  } else {
    const __half* p = static_cast<const __half*>(a.wscales) + (int64_t)u * a.N + n;
    for (int c = 0; c < cols; c += 64) prefetch_l1(p + c);
  }
}

// int4 units: the accumulators were seeded with the bit pattern of 1.5*2^23
// (kMagicBits), so each holds kMagicBits + acc; as a float that is exactly
// 1.5*2^23 + acc (|acc| < 2^22), and one subtraction gives F(acc) exactly.
// Same fp32 operations as fold8, two outputs per packed f32x2 instruction.
__device__ __forceinline__ void fold8_seeded(const uint32_t (&ap)[8], const uint32_t (&an)[8],
                                             const float (&sw)[8], float sp, float sn, float* y,
                                             float magic = kMagic) {
  const uint64_t m2 = f2_pack(-magic, -magic);
  const uint64_t sp2 = f2_pack(sp, sp), sn2 = f2_pack(sn, sn);
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const uint64_t fp = f2_add(f2_pack(__uint_as_float(ap[i]), __uint_as_float(ap[i + 1])), m2);
    const uint64_t fn = f2_add(f2_pack(__uint_as_float(an[i]), __uint_as_float(an[i + 1])), m2);
    const uint64_t t = f2_fma(sn2, fn, f2_mul(sp2, fp));
    const uint64_t yy = f2_fma(f2_pack(sw[i], sw[i + 1]), t, f2_pack(y[i], y[i + 1]));
    f2_unpack(yy, y[i], y[i + 1]);
  }
}

// int32 accumulator -> fp32, round to nearest even (an int8 unit's sum:
// |acc| <= 127 * 127 * K).
__device__ __forceinline__ float acc_f32(uint32_t v) { return __int2float_rn((int)v); }

// y (+)= sw * (s- F(acc-) + s+ F(acc+)) for eight columns, the fixed fp32
// order of fold8 on fp32 pairs (two outputs per packed instruction).
__device__ __forceinline__ void fold8_exact(const uint32_t (&ap)[8], const uint32_t (&an)[8],
                                            const float (&sw)[8], float sp, float sn, float* y) {
  const uint64_t sp2 = f2_pack(sp, sp), sn2 = f2_pack(sn, sn);
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const uint64_t fp = f2_pack(acc_f32(ap[i]), acc_f32(ap[i + 1]));
    const uint64_t fn = f2_pack(acc_f32(an[i]), acc_f32(an[i + 1]));
    const uint64_t yy = f2_fma(f2_pack(sw[i], sw[i + 1]), f2_fma(sn2, fn, f2_mul(sp2, fp)),
                               f2_pack(y[i], y[i + 1]));
    f2_unpack(yy, y[i], y[i + 1]);
  }
}

// Weight scales of 8 consecutive output channels for unit u, as four fp32 pairs.
__device__ __forceinline__ void load_wscales8_pairs(const GemmArgs& a, int u, int j, int n,
                                                    uint64_t (&sw2)[4]) {
  if (a.bits == 8) {
    const float4* s4 =
        reinterpret_cast<const float4*>(static_cast<const float*>(a.wscales) + (int64_t)j * a.N + n);
    const float4 t0 = __ldg(s4), t1 = __ldg(s4 + 1);
    sw2[0] = f2_pack(t0.x, t0.y); sw2[1] = f2_pack(t0.z, t0.w);
    sw2[2] = f2_pack(t1.x, t1.y); sw2[3] = f2_pack(t1.z, t1.w);
  } else {
    const uint4 t = __ldg(reinterpret_cast<const uint4*>(static_cast<const __half*>(a.wscales) +
                                                         (int64_t)u * a.N + n));
    const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
      sw2[k] = f2_pack(f.x, f.y);
    }
  }
}

// y2 (+)= sw * (s- F(acc-) + s+ F(acc+)) for 8 outputs held as four fp32 pairs,
// the same fp32 operations as fold8 (R9 order), two outputs per instruction.
// SEEDED: accumulators hold kMagicBits + acc (int4 units); F is one exact
// subtraction.  Otherwise F is the round-to-nearest int32 -> fp32 conversion.
template <bool SEEDED>
__device__ __forceinline__ void fold8_pairs(const uint32_t (&ap)[8], const uint32_t (&an)[8],
                                            const uint64_t (&sw2)[4], uint64_t sp2, uint64_t sn2,
                                            uint64_t* y2) {
  const uint64_t m2 = f2_pack(-kMagic, -kMagic);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint64_t fp, fn;
    if constexpr (SEEDED) {
      fp = f2_add(f2_pack(__uint_as_float(ap[2 * i]), __uint_as_float(ap[2 * i + 1])), m2);
      fn = f2_add(f2_pack(__uint_as_float(an[2 * i]), __uint_as_float(an[2 * i + 1])), m2);
    } else {
      fp = f2_pack(__int2float_rn((int)ap[2 * i]), __int2float_rn((int)ap[2 * i + 1]));
      fn = f2_pack(__int2float_rn((int)an[2 * i]), __int2float_rn((int)an[2 * i + 1]));
    }
    y2[i] = f2_fma(sw2[i], f2_fma(sn2, fn, f2_mul(sp2, fp)), y2[i]);
  }
}

// + bias, convert, two (bf16) or four (fp32) 16-byte stores.
template <bool Y_BF16>
__device__ __forceinline__ void store16(const GemmArgs& a, int row, int n, float (&o)[16]) {
  if (a.bias != nullptr) {
    const float4* b4 = reinterpret_cast<const float4*>(a.bias + n);
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
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.y) + (int64_t)row * a.ldy + n;
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(o[2 * i], o[2 * i + 1]);
      pk[i] = *reinterpret_cast<const uint32_t*>(&h2);
    }
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    reinterpret_cast<uint4*>(dst)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  } else {
    float* dst = static_cast<float*>(a.y) + (int64_t)row * a.ldy + n;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      reinterpret_cast<float4*>(dst)[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
  }
}

// --------------------------------------------------------- epilogue role
// Arrive on an mbarrier of another CTA of the cluster (release, cluster scope).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

// The epilogue of one CTA: for every tile it owns, wait for each unit's
// accumulators in TMEM, fold them (or write them raw), release the buffer,
// and after the tile's last unit store its rows.  The thread owns TMEM lane
// quad*32 + lane (tile row row_shift + quad*32 + lane) and the columns
// [part*HALF, (part+1)*HALF).  `empty_base` is the address of tmem_empty[0]
// (a cluster-window address of another CTA when empty_remote).
template <int BN, int NBUF, bool MULTI, bool ACC_OUT, bool Y_BF16, bool SEEDED, class TileFn,
          bool CLUSTER = false>
__device__ __forceinline__ void epilogue_role(const GemmArgs& args, int quad, int part, int lane,
                                              uint32_t t_lane, uint64_t* tmem_full,
                                              uint32_t empty_base, bool empty_remote,
                                              int row_shift, int rounds, TileFn tile_fn,
                                              volatile int* abort_flag, long long budget) {
  constexpr int HALF = BN / (epi_warps(MULTI) / 4);   // columns per epilogue thread
  const int half = part;
  const int num_kb = args.num_kb;
  const int units = (args.bits == 4) ? num_kb : args.kseg.count;
  auto release = [&](int b) {
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      if (empty_remote) mbar_arrive_remote(empty_base + 8u * (uint32_t)b);
      else mbar_arrive(empty_base + 8u * (uint32_t)b);
    }
  };
  int ug = 0;
  bool ok = true;
  if constexpr (SEEDED) {
    // Seed both accumulator buffers, then hand them to the MMA warp.
    const int c_lo = half * HALF;
    for (int b = 0; b < NBUF; ++b) {
#pragma unroll
      for (int c = 0; c < HALF / 8; ++c) {
        const uint32_t col = (uint32_t)(b * 2 * BN + c_lo + c * 8);
        tmem_st8(t_lane + col, kMagicBits);
        tmem_st8(t_lane + col + BN, kMagicBits);
      }
    }
    tmem_wait_st();
    for (int b = 0; b < NBUF; ++b) release(b);
  }
  for (int it = 0; it < rounds && ok; ++it) {
    Tile t;
    if (!tile_fn(it, t)) continue;
    const int row = t.m0 + row_shift + quad * 32 + lane;
    const int c_lo = half * HALF;                 // first tile column of this warp
      if constexpr (MULTI || ACC_OUT) {
        constexpr int NY2 = (MULTI && !ACC_OUT) ? HALF / 2 : 1;
        uint64_t y2[NY2];  // partial outputs, fp32 pairs
#pragma unroll
        for (int i = 0; i < NY2; ++i) y2[i] = 0ull;
        // Scales are read two units ahead of use, so their L2 latency hides
        // behind the current unit's MMAs.
        constexpr int kAhead = 2;
        if constexpr (!ACC_OUT) {
          if (lane == 0 && c_lo < t.width)
            for (int u = 0; u < kAhead && u < units; ++u)
              prefetch_wscales(args, u, (args.bits == 4) ? args.kseg.segment_of(u * 128) : u,
                               t.n0 + c_lo, min(HALF, t.width - c_lo));
        }
        for (int u = 0; u < units; ++u) {
          if constexpr (!ACC_OUT) {
            const int uf = u + kAhead;
            if (lane == 0 && uf < units && c_lo < t.width)
              prefetch_wscales(args, uf, (args.bits == 4) ? args.kseg.segment_of(uf * 128) : uf,
                               t.n0 + c_lo, min(HALF, t.width - c_lo));
          }
          const int b = ug % NBUF;
          if (!(ok = wait_warp<CLUSTER>(smem_u32(tmem_full + b), (ug / NBUF) & 1, abort_flag, budget))) break;
          tc_fence_after();
          const int j = (args.bits == 4) ? args.kseg.segment_of(u * 128) : u;
          const float sp = __ldg(args.s_pos + j), sn = __ldg(args.s_neg + j);
          const uint64_t sp2 = f2_pack(sp, sp), sn2 = f2_pack(sn, sn);
#pragma unroll
          for (int c = 0; c < HALF / 8; ++c) {
            if (c_lo + c * 8 < t.width) {
              uint32_t ap[8], an[8];
              const uint32_t col = (uint32_t)(b * 2 * BN + c_lo + c * 8);
              tmem_ld8(t_lane + col, ap);
              tmem_ld8(t_lane + col + BN, an);
              tmem_wait_ld();
              if constexpr (SEEDED) {
                tmem_st8(t_lane + col, kMagicBits);
                tmem_st8(t_lane + col + BN, kMagicBits);
              }
              const int n = t.n0 + c_lo + c * 8;
              if constexpr (ACC_OUT) {
                if constexpr (SEEDED) {
#pragma unroll
                  for (int i = 0; i < 8; ++i) { ap[i] -= kMagicBits; an[i] -= kMagicBits; }
                }
                if (row < args.M) {
                  int32_t* dp = args.acc_out + (((int64_t)u * 2 + 0) * args.M + row) * args.N + n;
                  int32_t* dn = args.acc_out + (((int64_t)u * 2 + 1) * args.M + row) * args.N + n;
#pragma unroll
                  for (int i = 0; i < 8; i += 4) {
                    *reinterpret_cast<uint4*>(dp + i) = make_uint4(ap[i], ap[i + 1], ap[i + 2], ap[i + 3]);
                    *reinterpret_cast<uint4*>(dn + i) = make_uint4(an[i], an[i + 1], an[i + 2], an[i + 3]);
                  }
                }
              } else {
                uint64_t sw2[4];
                load_wscales8_pairs(args, u, j, n, sw2);
                fold8_pairs<SEEDED>(ap, an, sw2, sp2, sn2, y2 + c * 4);
              }
            }
          }
          if constexpr (SEEDED) tmem_wait_st();
          release(b);
          ++ug;
        }
        if constexpr (!ACC_OUT) {
          if (ok && row < args.M) {
#pragma unroll
            for (int c = 0; c < HALF / 16; ++c) {
              if (c_lo + c * 16 < t.width) {
                float o[16];
#pragma unroll
                for (int i = 0; i < 8; ++i) f2_unpack(y2[c * 8 + i], o[2 * i], o[2 * i + 1]);
                store16<Y_BF16>(args, row, t.n0 + c_lo + c * 16, o);
              }
            }
          }
        }
      } else {
        // One unit per tile: stream column chunks from TMEM straight to memory.
        // The tile's scales and bias are fetched into L1 while its MMAs run.
        if (c_lo < t.width) {
          const int cols = min(HALF, t.width - c_lo);
          const float* sw_row = static_cast<const float*>(args.wscales) + t.n0 + c_lo;
          for (int c = lane * 32; c < cols; c += 32 * 32) prefetch_l1(sw_row + c);
          if (args.bias != nullptr)
            for (int c = lane * 32; c < cols; c += 32 * 32) prefetch_l1(args.bias + t.n0 + c_lo + c);
        }
        const int b = ug % NBUF;
        if (!(ok = wait_warp<CLUSTER>(smem_u32(tmem_full + b), (ug / NBUF) & 1, abort_flag, budget))) break;
        tc_fence_after();
        const float sp = __ldg(args.s_pos), sn = __ldg(args.s_neg);
#pragma unroll 1
        for (int c = 0; c < HALF / 16; ++c) {
          if (c_lo + c * 16 < t.width) {
            uint32_t ap[16], an[16];
            const uint32_t col = (uint32_t)(b * 2 * BN + c_lo + c * 16);
            tmem_ld16(t_lane + col, ap);
            tmem_ld16(t_lane + col + BN, an);
            tmem_wait_ld();
            if (row < args.M) {
              const int n = t.n0 + c_lo + c * 16;
              float sw[16], o[16];
              load_wscales16(args, 0, 0, n, sw);
#pragma unroll
              for (int i = 0; i < 16; ++i) o[i] = 0.0f;
              fold16<false>(ap, an, sw, sp, sn, o);
              store16<Y_BF16>(args, row, n, o);
            }
          }
        }
        release(b);
        ++ug;
      }
  }
}

// ------------------------------------------------- epilogue through TMA stores
// Output written by TMA tensor stores from a per-warp staging tile of 32 rows x
// 32 columns in shared memory.  Storing through TMA writes whole 128-byte lines
// instead of one 16-byte piece per row per lane, and the warp does not wait
// for the writes.
//
// Staging layout: row r (the warp's TMEM lane r) of the 32-column tile at
// r * ROWB, 16-byte chunk j of the row at position j ^ f(r) -- the TMA
// 64-byte swizzle for bf16 rows of 64 bytes (f(r) = (r >> 1) & 3) and the
// 128-byte swizzle for fp32 rows of 128 bytes (f(r) = r & 7) -- so a warp's
// 16-byte stores touch every bank evenly.  The buffer is 1024-byte aligned.
__host__ __device__ constexpr int stage_y_bytes(bool y_bf16) { return 32 * (y_bf16 ? 64 : 128); }

template <bool Y_BF16>
__device__ __forceinline__ void stage16(const GemmArgs& a, int n, float (&o)[16], uint8_t* srow,
                                        int r, int half) {
  if (a.bias != nullptr) {
    const float4* b4 = reinterpret_cast<const float4*>(a.bias + n);
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
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(o[2 * i], o[2 * i + 1]);
      pk[i] = *reinterpret_cast<const uint32_t*>(&h2);
    }
    const int f = (r >> 1) & 3;
    *reinterpret_cast<uint4*>(srow + (((2 * half) ^ f) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    *reinterpret_cast<uint4*>(srow + (((2 * half + 1) ^ f) << 4)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  } else {
    const int f = r & 7;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<float4*>(srow + (((4 * half + i) ^ f) << 4)) =
          make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
  }
}

// Single-scale fold of 16 columns: t = s * F(acc); y = fma(sw, t, y).
__device__ __forceinline__ void fold16_single(const uint32_t (&a)[16], const float (&sw)[16],
                                              float s, float* y) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float t = __fmul_rn(s, acc_to_f32<false>(a[i]));
    y[i] = __fmaf_rn(sw[i], t, y[i]);
  }
}

// Scale of unit u: the DualScale pair (s+, s-), or the single-scale s = max(s+, s-).
__device__ __forceinline__ void unit_act_scales(const GemmArgs& a, int j, float& sp, float& sn) {
  sp = __ldg(a.s_pos + j);
  sn = __ldg(a.s_neg + j);
}

// Epilogue warps: EPW of them; warp (quad, part) owns TMEM lanes quad*32..+31
// (tile rows) and columns [part*HALF, (part+1)*HALF).  NACC accumulators per
// unit (2: DualScale (+)/(-) products at columns c and c + BN of the buffer;
// 1: single scale).  MULTI: several units (K segments) per tile, folded into
// fp32 partial outputs in registers (HALF = 32 or 64 columns per thread),
// stored once per tile; otherwise one unit per tile, streamed out in
// 32-column passes.  Either way the accumulator buffer is released as soon as
// the warp's last TMEM load of the unit has landed, before the arithmetic on
// it, so the MMA of the next unit or tile waits only for the loads.
// (Group units -- one per 128-wide K group -- go through
// epilogue_groups_tma_store.)
// PAIR: a CTA of a 2-SM pair: its TMEM lanes are tile rows row_shift + 0..127,
// the full barriers are signalled by the leader's commits (cluster-scope
// acquire), and `empty_base` may be a cluster address of the leader's
// barriers (empty_remote).
// CSPLIT (one unit, two accumulators, four warps: the small-M two-tile form
// with the tile's k blocks split over the CTAs of a cluster): a CTA of rank
// r > 0 writes its raw accumulators into its own [2][128][BN] int32 buffer
// (`part`; accumulator a, lane quarter q, lane l, column c at
// ((128a + 32q + l) * BN + c) with the low five bits of c XOR l) and adds each
// warp's two 32-lane slices into the rank-0 CTA's buffer by bulk reductions
// counted on its `parts` barrier; rank 0 adds the buffer to its accumulators
// (integer sums, any order) before folding.
template <int BN, int NBUF, int EPW, int NACC, bool MULTI, bool Y_BF16, class TileFn,
          bool PAIR = false, bool CSPLIT = false, bool SPLIT = false>
__device__ __forceinline__ void epilogue_tma_store(const GemmArgs& args, const CUtensorMap* tmap_y,
                                                   uint8_t* stage_y, int quad, int part, int lane,
                                                   uint32_t t_lane, uint64_t* tmem_full,
                                                   uint32_t empty_base, int rounds, TileFn tile_fn,
                                                   volatile int* abort_flag, long long budget,
                                                   int row_shift = 0, bool empty_remote = false,
                                                   uint32_t crank = 0, uint32_t part_buf = 0,
                                                   uint32_t parts_bar = 0) {
  static_assert(!CSPLIT || (!MULTI && NACC == 2 && EPW == 4 && !PAIR), "K split: two-tile form");
  static_assert(!SPLIT || (BN == 256 && NBUF == 1 && EPW == 16 && NACC == 2 && !MULTI && !PAIR &&
                           !CSPLIT), "buffer released in halves: one 256-wide DualScale buffer");
  auto pidx = [&](int a, int c) {
    return (uint32_t)(((128 * a + quad * 32 + lane) * BN) + ((c & ~31) | ((c & 31) ^ lane)));
  };
  bool parts_in = false;
  bool sent = false;   // K split, rank > 0: this warp's slices have gone to rank 0
  constexpr int HALF = BN / (EPW / 4);
  constexpr int ROWB = Y_BF16 ? 64 : 128;
  constexpr uint32_t BUF_COLS = (uint32_t)(NACC * BN);
  static_assert(HALF % 32 == 0, "32-column store passes");
  static_assert(!MULTI || HALF <= 64, "several units: at most 64 partial outputs per thread");
  uint8_t* srow = stage_y + lane * ROWB;
  const uint32_t sbase = smem_u32(stage_y);
  const int units = args.kseg.count;
  auto release = [&](int b) {
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      if (PAIR && empty_remote) mbar_arrive_remote(empty_base + 8u * (uint32_t)b);
      else mbar_arrive(empty_base + 8u * (uint32_t)b);
    }
  };
  // Eight columns of buffer b at tile column cc into registers (both
  // polarities, or the single code's accumulator in ap).
  auto load8 = [&](int b, int cc, uint32_t (&ap)[8], uint32_t (&an)[8]) {
    const uint32_t tcol = (uint32_t)b * BUF_COLS + (uint32_t)cc;
    tmem_ld8(t_lane + tcol, ap);
    if constexpr (NACC == 2) tmem_ld8(t_lane + tcol + BN, an);
  };
  // y[0..8) (+)= the fold of eight loaded columns of unit / segment j
  auto fold8c = [&](const uint32_t (&ap)[8], const uint32_t (&an)[8], int j, int n, float sp,
                    float sn, float* y) {
    float sw[8];
    load_wscales8(args, j, j, n, sw);
    if constexpr (NACC == 2) {
      fold8_exact(ap, an, sw, sp, sn, y);
    } else {
      const float s = fmaxf(sp, sn);
#pragma unroll
      for (int i = 0; i < 8; ++i) y[i] = __fmaf_rn(sw[i], __fmul_rn(s, acc_f32(ap[i])), y[i]);
    }
  };
  int ug = 0;
  bool ok = true, pending = false;
  for (int it = 0; it < rounds && ok; ++it) {
    Tile t;
    if (!tile_fn(it, t)) continue;
    const int c_lo = part * HALF;
    const int cols = min(HALF, t.width - c_lo);   // may be <= 0 on a narrow tail tile
    if (SPLIT) {   // this warp's columns 32*part .. +32 and 128 + 32*part .. +32
      const int c0 = 128 * lane + 32 * part;
      if (lane < 2 && c0 < t.width) {
        prefetch_l1(static_cast<const float*>(args.wscales) + t.n0 + c0);
        if (args.bias != nullptr) prefetch_l1(args.bias + t.n0 + c0);
      }
    } else if (cols > 0) {
      for (int u = 0; u < (MULTI ? units : 1); ++u) {
        const float* sw_row = static_cast<const float*>(args.wscales) + (int64_t)u * args.N + t.n0 + c_lo;
        for (int c = lane * 32; c < cols; c += 32 * 32) prefetch_l1(sw_row + c);
      }
      if (args.bias != nullptr)
        for (int c = lane * 32; c < cols; c += 32 * 32) prefetch_l1(args.bias + t.n0 + c_lo + c);
    }
    const int npass = cols > 0 ? (cols + 31) / 32 : 0;
    // the number of eight-column chunks this warp folds (a multiple of 8 columns)
    const int nchunk = cols > 0 ? (cols + 7) / 8 : 0;
    if constexpr (MULTI) {
      float y[HALF];
#pragma unroll
      for (int i = 0; i < HALF; ++i) y[i] = 0.0f;
      for (int u = 0; u < units; ++u) {
        const int b = ug % NBUF;
        if (!(ok = wait_warp<PAIR>(smem_u32(tmem_full + b), (ug / NBUF) & 1, abort_flag, budget))) break;
        tc_fence_after();
        float sp, sn;
        unit_act_scales(args, u, sp, sn);
        bool released = false;
#pragma unroll
        for (int c = 0; c < HALF / 8; ++c) {
          if (c < nchunk) {
            uint32_t ap[8], an[8];
            load8(b, c_lo + 8 * c, ap, an);
            tmem_wait_ld();
            if (c + 1 == nchunk) {   // every column of the unit is in registers
              release(b);
              released = true;
            }
            fold8c(ap, an, u, t.n0 + c_lo + 8 * c, sp, sn, y + 8 * c);
          }
        }
        if (!released) release(b);
        ++ug;
      }
      if (!ok) break;
#pragma unroll
      for (int p = 0; p < HALF / 32; ++p) {
        if (p < npass) {
          if (pending) {   // the previous store has read the staging tile
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
          }
          const int col = c_lo + p * 32;
          stage16<Y_BF16>(args, t.n0 + col, *reinterpret_cast<float(*)[16]>(y + 32 * p), srow, lane, 0);
          if (col + 16 < t.width)
            stage16<Y_BF16>(args, t.n0 + col + 16, *reinterpret_cast<float(*)[16]>(y + 32 * p + 16),
                            srow, lane, 1);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(tmap_y, sbase, t.n0 + col, t.m0 + row_shift + quad * 32);
            bulk_commit_group();
          }
          pending = true;
        }
      }
    } else {
      const int b = ug % NBUF;
      if (!(ok = wait_warp<PAIR>(smem_u32(tmem_full + b), (ug / NBUF) & 1, abort_flag, budget))) break;
      tc_fence_after();
      float sp, sn;
      unit_act_scales(args, 0, sp, sn);
      // SPLIT: pass p covers tile columns 128p + 32*part .. +32, so every warp
      // reads the buffer's first half (both accumulators' columns 0 .. 127)
      // before the second, and hands each half back to the MMA on its own
      // barrier (tmem_empty[1]: first half; tmem_empty[0]: the whole buffer).
      const int np = SPLIT ? (32 * part < t.width ? 1 : 0) + (128 + 32 * part < t.width ? 1 : 0)
                           : npass;
      for (int p = 0; p < np; ++p) {
        const int col = SPLIT ? 128 * p + 32 * part : c_lo + p * 32;
        if (pending) {   // the previous store has read the staging tile
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int cc = col + 16 * h;
          if (cc < t.width) {
            uint32_t ap[8], an[8], bp[8], bn[8];
            load8(b, cc, ap, an);
            load8(b, cc + 8, bp, bn);
            tmem_wait_ld();
            if (h == 1 || cc + 16 >= t.width) {   // the pass's last loads
              if constexpr (SPLIT) {
                if (p == 0) release(1);
                if (p == np - 1) release(0);
              } else if (p == npass - 1) {
                release(b);
              }
            }
            if constexpr (CSPLIT) {
              uint32_t* pb = reinterpret_cast<uint32_t*>(__cvta_shared_to_generic(part_buf));
              if (crank != 0) {   // into this CTA's buffer; rank 0 folds
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                  pb[pidx(0, cc + k)] = ap[k];
                  pb[pidx(1, cc + k)] = an[k];
                  pb[pidx(0, cc + 8 + k)] = bp[k];
                  pb[pidx(1, cc + 8 + k)] = bn[k];
                }
                continue;
              }
              if (!parts_in) {   // the other CTAs' partial sums have landed
                if (!(ok = wait_warp<true>(parts_bar, 0, abort_flag, budget))) break;
                parts_in = true;
              }
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                ap[k] += pb[pidx(0, cc + k)];
                an[k] += pb[pidx(1, cc + k)];
                bp[k] += pb[pidx(0, cc + 8 + k)];
                bn[k] += pb[pidx(1, cc + 8 + k)];
              }
            }
            float o[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = 0.0f;
            fold8c(ap, an, 0, t.n0 + cc, sp, sn, o);
            fold8c(bp, bn, 0, t.n0 + cc + 8, sp, sn, o + 8);
            stage16<Y_BF16>(args, t.n0 + cc, o, srow, lane, h);
          }
        }
        if (!ok) break;
        if constexpr (CSPLIT) {
          if (crank != 0) {   // after the last pass: this warp's two slices into rank 0's buffer
            if (p == npass - 1) {
              fence_proxy_async_smem();   // the bulk copy reads through the async proxy
              __syncwarp();
              if (lane == 0) {
                const uint32_t part0 = mapa_shared(part_buf, 0), bar0 = mapa_shared(parts_bar, 0);
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                  const uint32_t off = (uint32_t)((128 * a + quad * 32) * BN * 4);
                  bulk_reduce_add_u32_cluster(part0 + off, part_buf + off, 32u * BN * 4u, bar0);
                }
              }
              sent = true;
            }
            continue;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(tmap_y, sbase, t.n0 + col, t.m0 + row_shift + quad * 32);
          bulk_commit_group();
        }
        pending = true;
      }
      if constexpr (SPLIT) {
        if (np == 0) {
          release(1);
          release(0);
        }
      } else if (npass == 0) {
        release(b);
      }
      ++ug;
    }
  }
  if constexpr (CSPLIT) {
    // After an abort the slices still go (their contents no longer count):
    // rank 0's barrier then completes, and rank 0 holds the cluster until
    // every add into its buffer has landed.
    if (crank != 0 && !sent) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const uint32_t part0 = mapa_shared(part_buf, 0), bar0 = mapa_shared(parts_bar, 0);
        for (int a = 0; a < 2; ++a) {
          const uint32_t off = (uint32_t)((128 * a + quad * 32) * BN * 4);
          bulk_reduce_add_u32_cluster(part0 + off, part_buf + off, 32u * BN * 4u, bar0);
        }
      }
    }
  }
  // Every store has completed before the CTA (and its shared memory) exits.
  if (lane == 0) bulk_wait_all();
  __syncwarp();
}

// ------------------------------------- stacked-polarity epilogue (small M)
// One row tile of P = args.a_rows rows (16, 32 or 64) whose codes were stacked
// in one A tile in groups of 16 rows: group g's q+ rows in A rows 32g .. +15,
// its q- rows in 32g + 16 .. +31.  The MMA therefore leaves the q+ product of
// tile row 16g + r in TMEM lane 32g + r and the q- product in lane 32g + 16 + r:
// epilogue warp g (lane quarter g, g < P/16) holds both halves of its 16 rows
// (the q- rows first, lanes 32g .. +15, when the codes map starts at q-).
// Each such warp prefetches the tile's weight scales and bias into L1 while
// the MMAs run, reads the whole tile from TMEM at once (BN/32 passes of 32
// columns in registers, one round trip) and releases it; per pass one exchange
// of 16 values gives lane l the (q+, q-) pair of row 16g + (l & 15), columns
// 16 * (l >> 4) .. +16, so all 32 lanes fold (fold8_exact: the outputs are
// those of the two-tile form); the passes stage into the warp's share of the
// eight 16-row staging tiles (`stage_y`: the four epilogue warps' 32 x 32
// tiles, halved) and leave by TMA stores of 16-row boxes (`tmap_y`), a batch
// at a time.
// CSPLIT (the tile's K range split over the CTAs of a cluster): in a CTA of
// rank r > 0 every warp holding accumulator lanes (TMEM lanes 0 .. 2P) writes
// its raw accumulators into its 32-lane slice of this CTA's [2P][BN] int32
// buffer (`part`, zeroed at setup; lane l of lane quarter q, column c, at
// (32q + l)*BN + c with the low five bits of c XOR l), then adds the slice into
// the rank-0 CTA's by one bulk reduction, counted as bytes on rank 0's `parts`
// barrier; rank 0's warps wait for every byte (bounded), add their slices to
// their own accumulators -- integer sums, exact in any order -- and fold and
// store as above.  (The buffers stay alive until rank 0 has seen every byte:
// the CTAs leave through a cluster barrier after the epilogue.  A warp that
// gave up on a wait still sends its slice, and rank 0, after giving up
// itself, waits for the bytes before that barrier, so no add lands in a CTA
// that has left.)
template <int BN, int NBUF, bool Y_BF16, bool CSPLIT = false, class TileFn>
__device__ __forceinline__ void epilogue_stacked(
    const GemmArgs& args, const CUtensorMap* tmap_y, uint8_t* stage_y, int quad, int lane,
    uint32_t t_lane, uint64_t* tmem_full, uint32_t empty_base, int rounds, TileFn tile_fn,
    volatile int* abort_flag, long long budget, uint32_t crank = 0, uint32_t part = 0,
    uint32_t parts_bar = 0) {
  static_assert(BN % 32 == 0 && BN <= 128, "32-column passes, at most four");
  constexpr int NPM = BN / 32;
  constexpr int ROWB = Y_BF16 ? 64 : 128;
  constexpr int SUB = 16 * ROWB;                                // one 16-row staging tile
  constexpr int NSUB = 4 * stage_y_bytes(Y_BF16) / SUB;         // eight
  // K split: this warp's 32 lanes of the [2P][BN] partial-sum buffer
  auto pidx = [&](int c) {
    return (uint32_t)((quad * 32 + lane) * BN + ((c & ~31) | ((c & 31) ^ lane)));
  };
  const uint32_t part0 = CSPLIT ? mapa_shared(part, 0) : 0u;   // rank 0's buffer
  bool parts_in = false;
  bool sent = false;   // rank > 0: this warp's slice has gone to rank 0
  const int groups = args.a_rows / 16;                          // warps holding rows
  const bool data_warp = quad < groups;
  const int ns = NSUB / groups;                                 // staging tiles per warp
  uint8_t* my_sub = stage_y + quad * ns * SUB;
  const bool hi = lane >= 16;
  const int r = lane & 15;                                      // row within the group
  const bool neg_first = args.code_box4 && args.code_neg_first;
  auto release = [&](int b) {
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_base + 8u * (uint32_t)b);
  };
  float sp, sn;
  unit_act_scales(args, 0, sp, sn);
  int ug = 0;
  bool ok = true, stored = false;
  for (int it = 0; it < rounds && ok; ++it) {
    Tile t;
    if (!tile_fn(it, t)) continue;
    // the tile's weight scales and bias into L1 while its MMAs run (a pass
    // would otherwise wait for them from HBM after the last MMA)
    if (data_warp && lane * 32 < t.width) {
      prefetch_l1(static_cast<const float*>(args.wscales) + t.n0 + lane * 32);
      if (args.bias != nullptr) prefetch_l1(args.bias + t.n0 + lane * 32);
    }
    const int b = ug % NBUF;
    if (!(ok = wait_warp(smem_u32(tmem_full + b), (ug / NBUF) & 1, abort_flag, budget))) break;
    tc_fence_after();
    ++ug;
    if (!data_warp) {   // lanes past 2P: nothing to read
      release(b);
      continue;
    }
    const int npass = (t.width + 31) / 32;
    // every column of the tile into registers at once, then the buffer released
    uint32_t va[NPM][4][8];
#pragma unroll
    for (int p = 0; p < NPM; ++p)
      if (p < npass)
#pragma unroll
        for (int i = 0; i < 4; ++i)
          tmem_ld8(t_lane + (uint32_t)b * BN + (uint32_t)(32 * p + 8 * i), va[p][i]);
    tmem_wait_ld();
    release(b);
    int first = 0;   // first pass of the batch being staged
#pragma unroll
    for (int p = 0; p < NPM; ++p) {
      if (p >= npass) break;
      const int col = 32 * p;
      uint32_t v[4][8];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int k = 0; k < 8; ++k) v[i][k] = va[p][i][k];
      if constexpr (CSPLIT) {
        if (crank != 0) {   // into this CTA's buffer, then added into rank 0's
          uint32_t* own = reinterpret_cast<uint32_t*>(__cvta_shared_to_generic(part));
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int k = 0; k < 8; ++k) own[pidx(col + 8 * i + k)] = v[i][k];
          if (p == npass - 1) {
            fence_proxy_async_smem();   // the bulk copy reads through the async proxy
            __syncwarp();
            if (lane == 0) {
              const uint32_t slice = (uint32_t)quad * 32u * BN * 4u;
              bulk_reduce_add_u32_cluster(part0 + slice, part + slice, 32u * BN * 4u,
                                          mapa_shared(parts_bar, 0));
            }
            sent = true;
          }
          continue;
        }
        if (!parts_in) {   // the other CTAs' partial sums have landed
          if (!(ok = wait_warp<true>(parts_bar, 0, abort_flag, budget))) break;
          parts_in = true;
        }
        const uint32_t* pb = reinterpret_cast<const uint32_t*>(__cvta_shared_to_generic(part));
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int k = 0; k < 8; ++k) v[i][k] += pb[pidx(col + 8 * i + k)];
      }
      // lane l: the (q+, q-) pair of row r, columns col + 16 * hi .. +16 --
      // the q- values of the first 16 columns go down to lanes 0-15, the q+
      // values of the last 16 up to lanes 16-31, picked without branching
      // (q- rows first in each group: the two halves swap roles)
      uint32_t fp[2][8], fn[2][8];
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t x = __shfl_xor_sync(0xffffffffu, hi ? v[i][k] : v[2 + i][k], 16);
          const uint32_t lo_half = hi ? x : v[i][k], hi_half = hi ? v[2 + i][k] : x;
          fp[i][k] = neg_first ? hi_half : lo_half;
          fn[i][k] = neg_first ? lo_half : hi_half;
        }
      // a new batch: the stores of the previous one have read their tiles
      if (p == first && stored) {
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
      }
      uint8_t* sub = my_sub + (p - first) * SUB;
      const int h = hi ? 1 : 0;
      const int cc = col + 16 * h;
      if (cc < t.width) {
        float o[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] = 0.0f;
        float sw[8];
        load_wscales8(args, 0, 0, t.n0 + cc, sw);
        fold8_exact(fp[0], fn[0], sw, sp, sn, o);
        load_wscales8(args, 0, 0, t.n0 + cc + 8, sw);
        fold8_exact(fp[1], fn[1], sw, sp, sn, o + 8);
        stage16<Y_BF16>(args, t.n0 + cc, o, sub + r * ROWB, r, h);
      }
      // the batch leaves when the warp's tiles are full or the tile is done
      if (p - first == ns - 1 || p == npass - 1) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          for (int q = first; q <= p; ++q)
            tma_store_2d(tmap_y, smem_u32(my_sub + (q - first) * SUB), t.n0 + 32 * q,
                         t.m0 + 16 * quad);
          bulk_commit_group();
        }
        stored = true;
        first = p + 1;
      }
    }
  }
  if constexpr (CSPLIT) {
    // After an abort the slice still goes (its contents no longer count):
    // rank 0's barrier then completes, and rank 0 holds the cluster until
    // every add into its buffer has landed.
    if (crank != 0 && data_warp && !sent) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const uint32_t slice = (uint32_t)quad * 32u * BN * 4u;
        bulk_reduce_add_u32_cluster(part0 + slice, part + slice, 32u * BN * 4u,
                                    mapa_shared(parts_bar, 0));
      }
    }
  }
  // Every store has completed before the CTA (and its shared memory) exits.
  if (lane == 0) bulk_wait_all();
  __syncwarp();
}

// ------------------------------------------- group-unit epilogue (int4 groups)
// One unit per 128-wide K group (int4 weights, SEED 1; the Hadamard-rotated
// codes, SEED 2): every k block ends a unit, so the whole accumulator pair is
// folded once per 512 tensor-core cycles and the fold's instruction count sets
// the kernel's speed.  Warp (quad, part) owns TMEM lanes quad*32 .. +31 (tile
// rows) and the 32 columns [part*32, part*32 + 32) of every group:
//   * the group's fp16 weight scales of those columns are widened to fp32 once
//     per lane (lane l: column l, fetched one group ahead) and staged in the
//     warp's shared-memory slot `sw_stage` (two buffers of 32 floats,
//     alternating by group), from which every lane reads them back with
//     broadcast 16-byte loads;
//   * the accumulators (seeded by the unit's first MMA) are read eight
//     columns at a time per polarity, and the buffer goes back to the MMA as
//     soon as its last columns are in registers; F(acc) is one exact
//     subtraction (the seed's bits plus the integer sum are the float seed +
//     acc);
//   * the fold runs on fp32 pairs, five packed instructions per two outputs,
//     in the fixed order t = fma(s-, F-, s+ * F+), y = fma(sw, t, y), y from 0.
// After the tile's last group: + bias, convert, TMA store of the warp's
// 32 x 32 block from its staging tile.
template <int EPW, bool Y_BF16, int SEED, class TileFn>
__device__ __forceinline__ void epilogue_groups_tma_store(
    const GemmArgs& args, const CUtensorMap* tmap_y, uint8_t* stage_y, float* sw_stage, int quad,
    int part, int lane, uint32_t t_lane, uint64_t* tmem_full, uint32_t empty_base, int rounds,
    TileFn tile_fn, volatile int* abort_flag, long long budget) {
  constexpr int BN = 128;
  constexpr int NBUF = 2;
  static_assert(EPW == 16, "four parts of 32 columns per lane quarter");
  static_assert(SEED == 1 || SEED == 2, "seeded group units");
  constexpr uint32_t BUF_COLS = 2u * BN;
  constexpr float seed_value = (SEED == 1) ? kMagicW4 : kMagic;
  constexpr float act_mult = (SEED == 2) ? 0.25f : 1.0f;   // Hadamard block normalization
  constexpr int ROWB = Y_BF16 ? 64 : 128;
  uint8_t* srow = stage_y + lane * ROWB;
  const uint32_t sbase = smem_u32(stage_y);
  const int G = args.num_kb;
  const int c_lo = part * 32;
  const __half* wsc = static_cast<const __half*>(args.wscales);
  const uint64_t mseed = f2_pack(-seed_value, -seed_value);
  auto release = [&](int b) {
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_base + 8u * (uint32_t)b);
  };
  int ug = 0;
  bool ok = true, pending = false;
  for (int it = 0; it < rounds && ok; ++it) {
    Tile t;
    if (!tile_fn(it, t)) continue;
    const bool active = c_lo < t.width;                 // warp-uniform
    const bool n_ok = active && (c_lo + lane < t.width);
    const __half* wcol = wsc + t.n0 + c_lo + lane;      // this lane's column, group 0
    const __half hzero = __ushort_as_half((unsigned short)0);
    // group 0's scales staged now, group 1's fetched
    sw_stage[lane] = __half2float(n_ok ? __ldg(wcol) : hzero);
    __half h_next = (n_ok && G > 1) ? __ldg(wcol + args.N) : hzero;
    __syncwarp();
    uint64_t y2[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) y2[i] = 0ull;
    int j = 0;
    int seg_end = args.kseg.b[1];
    float sp = __fmul_rn(__ldg(args.s_pos), act_mult), sn = __fmul_rn(__ldg(args.s_neg), act_mult);
    uint64_t sp2 = f2_pack(sp, sp), sn2 = f2_pack(sn, sn);
    for (int u = 0; u < G; ++u) {
      if (u * BK >= seg_end) {   // the group opens the next K segment
        ++j;
        seg_end = args.kseg.b[j + 1];
        sp = __fmul_rn(__ldg(args.s_pos + j), act_mult);
        sn = __fmul_rn(__ldg(args.s_neg + j), act_mult);
        sp2 = f2_pack(sp, sp);
        sn2 = f2_pack(sn, sn);
      }
      const int b = ug % NBUF;
      if (!(ok = wait_warp(smem_u32(tmem_full + b), (ug / NBUF) & 1, abort_flag, budget))) break;
      tc_fence_after();
      if (active) {
        const float* sw = sw_stage + (u & 1) * 32;
#pragma unroll
        for (int h = 0; h < 4; ++h) {   // eight columns at a time (register budget)
          const uint32_t col = (uint32_t)b * BUF_COLS + (uint32_t)(c_lo + 8 * h);
          uint32_t ap[8], an[8];
          tmem_ld8(t_lane + col, ap);
          tmem_ld8(t_lane + col + BN, an);
          tmem_wait_ld();
          if (h == 3) release(b);   // the group's last columns are in registers
          const float4* s4 = reinterpret_cast<const float4*>(sw + 8 * h);
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const float4 s = s4[q];
            const uint64_t sw_lo = f2_pack(s.x, s.y), sw_hi = f2_pack(s.z, s.w);
            const int i = 4 * q;
            // F(acc): one exact subtraction per accumulator, packed for int4
            // weights, scalar for the Hadamard-rotated codes (each measured
            // faster for its kernel)
            uint64_t fp0, fn0, fp1, fn1;
            if constexpr (SEED == 1) {
              fp0 = f2_add(f2_pack(__uint_as_float(ap[i]), __uint_as_float(ap[i + 1])), mseed);
              fn0 = f2_add(f2_pack(__uint_as_float(an[i]), __uint_as_float(an[i + 1])), mseed);
              fp1 = f2_add(f2_pack(__uint_as_float(ap[i + 2]), __uint_as_float(ap[i + 3])), mseed);
              fn1 = f2_add(f2_pack(__uint_as_float(an[i + 2]), __uint_as_float(an[i + 3])), mseed);
            } else {
              fp0 = f2_pack(__fadd_rn(__uint_as_float(ap[i]), -seed_value),
                            __fadd_rn(__uint_as_float(ap[i + 1]), -seed_value));
              fn0 = f2_pack(__fadd_rn(__uint_as_float(an[i]), -seed_value),
                            __fadd_rn(__uint_as_float(an[i + 1]), -seed_value));
              fp1 = f2_pack(__fadd_rn(__uint_as_float(ap[i + 2]), -seed_value),
                            __fadd_rn(__uint_as_float(ap[i + 3]), -seed_value));
              fn1 = f2_pack(__fadd_rn(__uint_as_float(an[i + 2]), -seed_value),
                            __fadd_rn(__uint_as_float(an[i + 3]), -seed_value));
            }
            y2[4 * h + 2 * q] = f2_fma(sw_lo, f2_fma(sn2, fn0, f2_mul(sp2, fp0)), y2[4 * h + 2 * q]);
            y2[4 * h + 2 * q + 1] = f2_fma(sw_hi, f2_fma(sn2, fn1, f2_mul(sp2, fp1)), y2[4 * h + 2 * q + 1]);
          }
        }
      } else {
        release(b);
      }
      ++ug;
      if (u + 1 < G) {   // stage group u+1's scales (its buffer was last read in group u-1)
        sw_stage[((u + 1) & 1) * 32 + lane] = __half2float(h_next);
        h_next = (n_ok && u + 2 < G) ? __ldg(wcol + (int64_t)(u + 2) * args.N) : hzero;
        __syncwarp();
      }
    }
    if (!ok) break;
    if (active) {
      if (pending) {   // the previous store has read the staging tile
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
      }
      float o[32];
#pragma unroll
      for (int i = 0; i < 16; ++i) f2_unpack(y2[i], o[2 * i], o[2 * i + 1]);
      stage16<Y_BF16>(args, t.n0 + c_lo, *reinterpret_cast<float(*)[16]>(o), srow, lane, 0);
      if (c_lo + 16 < t.width)
        stage16<Y_BF16>(args, t.n0 + c_lo + 16, *reinterpret_cast<float(*)[16]>(o + 16), srow, lane, 1);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(tmap_y, sbase, t.n0 + c_lo, t.m0 + quad * 32);
        bulk_commit_group();
      }
      pending = true;
    }
  }
  // Every store has completed before the CTA (and its shared memory) exits.
  if (lane == 0) bulk_wait_all();
  __syncwarp();
}

// ------------------------------------------------------------------ kernel
// MULTI: more than one unit per tile (several K segments, or int4 groups):
// partial outputs stay in registers across units (BN = 128 only, 16 epilogue
// warps).
template <int BN, int ASRC, typename XT, bool W4, bool ACC_OUT, bool Y_BF16, bool MULTI>
__global__ void __launch_bounds__(kernel_threads(MULTI), 1)
    dualscale_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                          const __grid_constant__ CUtensorMap tmap_a2,
                          const __grid_constant__ CUtensorMap tmap_w,
                          const __grid_constant__ GemmArgs args) {
  using C = GemmCfg<BN, ASRC, XT, W4>;
  static_assert(!MULTI || BN == 128, "several units per tile need double-buffered TMEM");
  static_assert(!W4 || MULTI, "int4 weights fold one unit per 128-wide group");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sm_x = smem + C::OFF_X;
  uint8_t* sm_wp = smem + C::OFF_WP;
  uint8_t* sm_w = smem + C::OFF_W;
  uint8_t* sm_q = smem + C::OFF_Q;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full_x = bars;                 // [2]
  uint64_t* empty_x = full_x + 2;          // [2]
  uint64_t* full_wp = empty_x + 2;         // [4]
  uint64_t* empty_wp = full_wp + 4;        // [4]
  uint64_t* full_w = empty_wp + 4;         // [4]
  uint64_t* empty_w = full_w + 4;          // [4]
  uint64_t* full_q = empty_w + 4;          // [8]
  uint64_t* empty_q = full_q + 8;          // [8]
  uint64_t* tmem_full = empty_q + 8;       // [2]
  uint64_t* tmem_empty = tmem_full + 2;    // [2]
  uint64_t* drain_bar = tmem_empty + 2;    // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long budget = args.wait_budget;
  constexpr bool PROD_Q = (ASRC == ASRC_X);   // producer warps write the Q tiles
  constexpr bool PROD_W = W4;                 // producer warps write the W tiles
  constexpr bool SEEDED = W4;                 // accumulators seeded with kMagicBits

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::SX; ++i) {
      mbar_init(smem_u32(full_x + i), 1);
      mbar_init(smem_u32(empty_x + i), kProdWarps);
    }
    for (int i = 0; i < C::SWP; ++i) {
      mbar_init(smem_u32(full_wp + i), 1);
      mbar_init(smem_u32(empty_wp + i), kProdWarps);
    }
    for (int i = 0; i < C::SW; ++i) {
      mbar_init(smem_u32(full_w + i), PROD_W ? kProdWarps : 1);
      mbar_init(smem_u32(empty_w + i), 1);
    }
    for (int i = 0; i < C::SQ; ++i) {
      mbar_init(smem_u32(full_q + i), PROD_Q ? kProdWarps : 1);
      mbar_init(smem_u32(empty_q + i), 1);
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

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_a);
      if constexpr (ASRC == ASRC_CODES) tma_prefetch_desc(&tmap_a2);
      tma_prefetch_desc(&tmap_w);
      int ca = 0, cw = 0;
      bool ok = (args.starve == 0);
      for (int it = 0; it < rounds && ok; ++it) {
        Tile t;
        if (!tile_of(args, it, BN, t)) continue;
        for (int kb = 0; kb < num_kb; ++kb) {
          if constexpr (ASRC == ASRC_X) {
            const int s = ca % C::SX;
            if (!(ok = wait1(smem_u32(empty_x + s), ((ca / C::SX) & 1) ^ 1, abort_flag, budget))) break;
            mbar_arrive_expect_tx(smem_u32(full_x + s), C::X_STAGE);
            for (int b = 0; b < C::X_BOXES; ++b)
              tma_load_2d(smem_u32(sm_x + s * C::X_STAGE + b * C::X_BOX_BYTES), &tmap_a,
                          smem_u32(full_x + s), kb * BK + b * C::X_EPB, t.m0);
          } else {
            const int s = ca % C::SQ;
            if (!(ok = wait1(smem_u32(empty_q + s), ((ca / C::SQ) & 1) ^ 1, abort_flag, budget))) break;
            mbar_arrive_expect_tx(smem_u32(full_q + s), C::Q_STAGE);
            tma_load_2d(smem_u32(sm_q + s * C::Q_STAGE), &tmap_a, smem_u32(full_q + s), kb * BK, t.m0);
            tma_load_2d(smem_u32(sm_q + s * C::Q_STAGE + C::Q_TILE), &tmap_a2, smem_u32(full_q + s),
                        kb * BK, t.m0);
          }
          ++ca;
          if constexpr (W4) {
            const int s = cw % C::SWP;
            if (!(ok = wait1(smem_u32(empty_wp + s), ((cw / C::SWP) & 1) ^ 1, abort_flag, budget))) break;
            mbar_arrive_expect_tx(smem_u32(full_wp + s), C::WP_STAGE);
            tma_load_2d(smem_u32(sm_wp + s * C::WP_STAGE), &tmap_w, smem_u32(full_wp + s),
                        kb * (BK / 2), t.n0);
          } else {
            const int s = cw % C::SW;
            if (!(ok = wait1(smem_u32(empty_w + s), ((cw / C::SW) & 1) ^ 1, abort_flag, budget))) break;
            mbar_arrive_expect_tx(smem_u32(full_w + s), C::W_STAGE);
            tma_load_2d(smem_u32(sm_w + s * C::W_STAGE), &tmap_w, smem_u32(full_w + s), kb * BK, t.n0);
          }
          ++cw;
        }
      }
      // Let every copy this thread started land before the CTA can exit.
      if constexpr (ASRC == ASRC_X) drain_ring(full_x, C::SX, ca, kDrainBudget);
      else drain_ring(full_q, C::SQ, ca, kDrainBudget);
      if constexpr (W4) drain_ring(full_wp, C::SWP, cw, kDrainBudget);
      else drain_ring(full_w, C::SW, cw, kDrainBudget);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int cq = 0, cw = 0, ug = 0;
      bool ok = true;
      for (int it = 0; it < rounds && ok; ++it) {
        Tile t;
        if (!tile_of(args, it, BN, t)) continue;
        const uint32_t idesc = idesc_i8(BM, t.width);
        bool unit_open = false;
        uint32_t d_pos = 0;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!unit_open) {
            const int b = ug % C::NBUF;
            // Seeded (int4) accumulators: the epilogue's seeding of a buffer
            // completes phase 0, so use n waits for phase n; otherwise a fresh
            // buffer is free at once.
            const uint32_t par = SEEDED ? ((ug / C::NBUF) & 1) : (((ug / C::NBUF) & 1) ^ 1);
            if (!(ok = wait1(smem_u32(tmem_empty + b), par, abort_flag, budget))) break;
            tc_fence_after();
            d_pos = tmem_base + (uint32_t)(b * 2 * BN);
          }
          const int sw = cw % C::SW, sq = cq % C::SQ;
          if (!(ok = wait1(smem_u32(full_w + sw), (cw / C::SW) & 1, abort_flag, budget))) break;
          if (!(ok = wait1(smem_u32(full_q + sq), (cq / C::SQ) & 1, abort_flag, budget))) break;
          tc_fence_after();
          const uint32_t a_p = smem_u32(sm_q + sq * C::Q_STAGE);
          const uint32_t a_n = a_p + C::Q_TILE;
          const uint32_t b_w = smem_u32(sm_w + sw * C::W_STAGE);
#pragma unroll
          for (int ks = 0; ks < BK / 32; ++ks) {
            const uint32_t acc = (SEEDED || unit_open || ks > 0) ? 1u : 0u;
            const uint64_t bd = smem_desc_k_sw128(b_w + ks * 32);
            umma_i8(d_pos, smem_desc_k_sw128(a_p + ks * 32), bd, idesc, acc);
            umma_i8(d_pos + BN, smem_desc_k_sw128(a_n + ks * 32), bd, idesc, acc);
          }
          unit_open = true;
          umma_commit(smem_u32(empty_w + sw));
          umma_commit(smem_u32(empty_q + sq));
          ++cw;
          ++cq;
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
  } else if (warp < kEpiWarp0) {
    // ------------------------------------------------- operand producers
    if constexpr (PROD_Q || PROD_W) {
      const int t_id = threadIdx.x - kProdWarp0 * 32;  // 0..255
      const int row = t_id & (BM - 1);                 // tile row (quantizer)
      const int c0 = (t_id >> 7) * 4;                  // first of its four 16-wide chunks
      int cx = 0, cq = 0, cwp = 0, cw = 0;
      int cur_seg = -1;
      QuantParams qpar{0.0f, 0u, 0u};
      bool ok = true;
      for (int it = 0; it < rounds && ok; ++it) {
        Tile t;
        if (!tile_of(args, it, BN, t)) continue;
        for (int kb = 0; kb < num_kb; ++kb) {
          if constexpr (PROD_Q) {
            const int j = kb_segment(args, kb);
            if (j != cur_seg) {
              cur_seg = j;
              qpar = quant_params(__ldg(args.s_pos + j), __ldg(args.s_neg + j));
            }
            const int sx = cx % C::SX, sq = cq % C::SQ;
            if (!(ok = wait_warp(smem_u32(full_x + sx), (cx / C::SX) & 1, abort_flag, budget))) break;
            if (!(ok = wait_warp(smem_u32(empty_q + sq), ((cq / C::SQ) & 1) ^ 1, abort_flag, budget))) break;
            const uint8_t* xs = sm_x + sx * C::X_STAGE;
            uint8_t* qp = sm_q + sq * C::Q_STAGE + row * 128;
            uint8_t* qn = qp + C::Q_TILE;
#pragma unroll 2
            for (int c = c0; c < c0 + 4; ++c) {
              float v[16];
              load_row16<XT>(xs, row, c, v);
              uint4 up, un;
              quantize16_fast(v, qpar, up, un);
              const int off = (c ^ (row & 7)) << 4;
              *reinterpret_cast<uint4*>(qp + off) = up;
              *reinterpret_cast<uint4*>(qn + off) = un;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(empty_x + sx));
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(full_q + sq));
            ++cx;
            ++cq;
          }
          if constexpr (PROD_W) {
            const int sp_ = cwp % C::SWP, sw = cw % C::SW;
            if (!(ok = wait_warp(smem_u32(full_wp + sp_), (cwp / C::SWP) & 1, abort_flag, budget))) break;
            if (!(ok = wait_warp(smem_u32(empty_w + sw), ((cw / C::SW) & 1) ^ 1, abort_flag, budget))) break;
            const uint8_t* src = sm_wp + sp_ * C::WP_STAGE;
            uint8_t* dst = sm_w + sw * C::W_STAGE;
#pragma unroll
            for (int i = 0; i < (BN * 4) / (kProdWarps * 32); ++i) {
              const int task = i * (kProdWarps * 32) + t_id;
              const int n = task >> 2, q = task & 3;   // row, 16-byte quarter of the packed row
              const uint4 pk = *reinterpret_cast<const uint4*>(src + n * 64 + q * 16);
              const uint2 e0 = unpack8_int4(pk.x), e1 = unpack8_int4(pk.y);
              const uint2 e2 = unpack8_int4(pk.z), e3 = unpack8_int4(pk.w);
              uint8_t* drow = dst + n * 128;
              *reinterpret_cast<uint4*>(drow + (((2 * q) ^ (n & 7)) << 4)) = make_uint4(e0.x, e0.y, e1.x, e1.y);
              *reinterpret_cast<uint4*>(drow + (((2 * q + 1) ^ (n & 7)) << 4)) = make_uint4(e2.x, e2.y, e3.x, e3.y);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(empty_wp + sp_));
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(full_w + sw));
            ++cwp;
            ++cw;
          }
        }
      }
    }
  } else {
    // --------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int part = (warp - kEpiWarp0) >> 2;
    epilogue_role<BN, C::NBUF, MULTI, ACC_OUT, Y_BF16, SEEDED>(
        args, quad, part, lane, tmem_base + ((uint32_t)(quad * 32) << 16), tmem_full,
        smem_u32(tmem_empty), /*empty_remote=*/false, /*row_shift=*/0, rounds,
        [&](int it, Tile& t) { return tile_of(args, it, BN, t); }, abort_flag, budget);
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
