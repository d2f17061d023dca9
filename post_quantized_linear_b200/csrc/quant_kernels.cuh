// HBM-bound DualScale kernels: static calibration (per-segment polarity
// maxima), standalone activation quantization, and weight quantization
// (int8 per channel and K segment, int4 group-128 with fp16 scales).
//
// SegQuant ("SegQuant: A Semantics-Aware and Generalizable Quantization
// Framework for Diffusion Models"): DualScale splits X into non-negative and
// negative parts with separate static scales (Spanish technical summary 2.B,
// Korean technical summary section 2 "DualScale"); SegLinear gives each input
// segment its own scales (Spanish technical summary 2.A).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"

namespace sq {

// ----------------------------------------------------------------- loads
// 16-byte vector of activations widened to fp32: 8 bf16 or 4 fp32 values.
template <typename XT> struct Vec;
template <> struct Vec<__nv_bfloat16> {
  static constexpr int n = 8;
  __device__ __forceinline__ static void load(const void* p, float (&v)[8]) {
    load_raw(__ldg(reinterpret_cast<const uint4*>(p)), v);
  }
  __device__ __forceinline__ static void load_raw(const uint4& u, float (&v)[8]) {
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};
template <> struct Vec<float> {
  static constexpr int n = 4;
  __device__ __forceinline__ static void load(const void* p, float (&v)[4]) {
    float4 u = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  }
  __device__ __forceinline__ static void load_raw(const uint4& u, float (&v)[4]) {
    v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y);
    v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
  }
};

// ------------------------------------------------------------ calibration
// blockDim = (32, 8).  Lane x of the block owns the 16-byte column vector
// v = blockIdx.x * 32 + x of every row it visits (rows blockIdx.y*8+y, stepping
// by gridDim.y*8), so each thread sees one K segment only.  Groups of 16 lanes
// cover 128 bf16 / 64 fp32 columns, never straddling a segment bound (bounds
// are multiples of 128), so a 16-lane shuffle reduction is exact.  Block
// maxima are combined in shared memory, then divided by 127 and merged into
// the outputs with an integer atomicMax on the fp32 bit patterns: for
// non-negative floats the bit order is the value order, and rounding the
// quotient is monotone, so max_c(fl(P_c/127)) = fl(max_c P_c / 127).
// The outputs must be zeroed before the launch.
template <typename XT>
__global__ void __launch_bounds__(256) calibrate_kernel(const XT* __restrict__ x, int64_t rows,
                                                        int64_t K, int64_t ldx, SegBounds kseg,
                                                        float* __restrict__ s_pos,
                                                        float* __restrict__ s_neg) {
  constexpr int VN = Vec<XT>::n;
  __shared__ unsigned int sh_p[SQ_MAX_SEG], sh_n[SQ_MAX_SEG];
  __shared__ int sh_bad;
  const int tid = threadIdx.y * 32 + threadIdx.x;
  if (tid < SQ_MAX_SEG) { sh_p[tid] = 0u; sh_n[tid] = 0u; }
  if (tid == 0) sh_bad = 0;
  __syncthreads();

  const int64_t nvec = K / VN;
  const int64_t v = (int64_t)blockIdx.x * 32 + threadIdx.x;
  const bool active = v < nvec;
  const int j = active ? kseg.segment_of((int32_t)(v * VN)) : 0;
  float P = 0.0f, Q = 0.0f;
  bool bad = false;
  if (active) {
    const XT* col = x + v * VN;
    int64_t m = (int64_t)blockIdx.y * 8 + threadIdx.y;
    const int64_t step = (int64_t)gridDim.y * 8;
    // eight rows in flight per thread, kept as raw 16-byte vectors
    for (; m + 7 * step < rows; m += 8 * step) {
      uint4 raw[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        raw[u] = __ldg(reinterpret_cast<const uint4*>(col + (m + u * step) * ldx));
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        float a[VN];
        Vec<XT>::load_raw(raw[u], a);
#pragma unroll
        for (int i = 0; i < VN; ++i) {
          const float t = a[i];
          bad |= (t != t) || (fabsf(t) == __int_as_float(0x7f800000));
          P = fmaxf(P, t);
          Q = fmaxf(Q, -t);
        }
      }
    }
    for (; m + 3 * step < rows; m += 4 * step) {
      float a[4][VN];
#pragma unroll
      for (int u = 0; u < 4; ++u) Vec<XT>::load(col + (m + u * step) * ldx, a[u]);
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int i = 0; i < VN; ++i) {
          const float t = a[u][i];
          bad |= (t != t) || (fabsf(t) == __int_as_float(0x7f800000));
          P = fmaxf(P, t);
          Q = fmaxf(Q, -t);
        }
    }
    for (; m < rows; m += step) {
      float a[VN];
      Vec<XT>::load(col + m * ldx, a);
#pragma unroll
      for (int i = 0; i < VN; ++i) {
        bad |= (a[i] != a[i]) || (fabsf(a[i]) == __int_as_float(0x7f800000));
        P = fmaxf(P, a[i]);
        Q = fmaxf(Q, -a[i]);
      }
    }
  }
  // 16-lane max reduction (all 16 lanes share one segment).
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) {
    P = fmaxf(P, __shfl_xor_sync(0xffffffffu, P, o));
    Q = fmaxf(Q, __shfl_xor_sync(0xffffffffu, Q, o));
  }
  const unsigned any_bad = __ballot_sync(0xffffffffu, bad);
  if (active && (threadIdx.x & 15) == 0) {
    atomicMax(&sh_p[j], __float_as_uint(P));
    atomicMax(&sh_n[j], __float_as_uint(Q));
  }
  if (threadIdx.x == 0 && any_bad) sh_bad = 1;
  __syncthreads();
  if (tid < kseg.count) {
    const float p = __uint_as_float(sh_p[tid]) / 127.0f;
    const float q = __uint_as_float(sh_n[tid]) / 127.0f;
    if (p > 0.0f) atomicMax(reinterpret_cast<unsigned int*>(s_pos) + tid, __float_as_uint(p));
    if (q > 0.0f) atomicMax(reinterpret_cast<unsigned int*>(s_neg) + tid, __float_as_uint(q));
  }
  if (tid == 0 && sh_bad) raise_status(SQ_STATUS_RANGE);
}

// ------------------------------------------------------- DualScale codes
// q+ = clamp(rne(max(x,0) * r+), 0, 127), q- = clamp(rne(min(x,0) * r-), -127, 0).
// The rounding adds the exact product to 1.5 * 2^23 in one fma: in
// [2^23, 2^24) the fp32 spacing is 1, so the fma's round-half-even lands on
// 1.5*2^23 + rne(x*r) (the offset is even, so ties still go to even), and the
// code is the low byte of the bit pattern.  Out-of-range sums are clamped in
// the float domain first (fmin/fmax are monotone, so clamping commutes with
// the rounding).
__device__ __forceinline__ uint32_t code_pos(float v, float r) {
  const float t = fminf(fmaf(fmaxf(v, 0.0f), r, kMagic), kMagic + 127.0f);
  return __float_as_uint(t);
}
__device__ __forceinline__ uint32_t code_neg(float v, float r) {
  const float t = fmaxf(fmaf(fminf(v, 0.0f), r, kMagic), kMagic - 127.0f);
  return __float_as_uint(t);
}
// Low bytes of four fp32 bit patterns into one word (byte i from a_i).
__device__ __forceinline__ uint32_t pack4_low(uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3) {
  const uint32_t lo = __byte_perm(a0, a1, 0x0040);
  const uint32_t hi = __byte_perm(a2, a3, 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}

// Loads 16 consecutive activations widened to fp32 (two bf16 or four fp32
// 16-byte vectors).
template <typename XT>
__device__ __forceinline__ void load16(const XT* p, float (&v)[16]) {
  if constexpr (Vec<XT>::n == 8) {
    float a[8], b[8];
    Vec<XT>::load(p, a);
    Vec<XT>::load(p + 8, b);
#pragma unroll
    for (int i = 0; i < 8; ++i) { v[i] = a[i]; v[8 + i] = b[i]; }
  } else {
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      float a[4];
      Vec<XT>::load(p + 4 * h, a);
#pragma unroll
      for (int i = 0; i < 4; ++i) v[4 * h + i] = a[i];
    }
  }
}

// ------------------------------------------------ block Hadamard transform
// HQ-DM ("HQ-DM: Single Hadamard Transformation-Based Quantization-Aware
// Training for Low-Bit Diffusion Models", Spanish technical summary 2.1): the
// activations are multiplied by a block-diagonal Hadamard matrix before they
// are quantized.  Blocks of 16 along K: the Sylvester-ordered butterfly (stage
// h = 1, 2, 4, 8: (v[j], v[j+h]) -> (v[j] + v[j+h], v[j] - v[j+h]), each
// rounded to fp32), then the normalization 1/sqrt(16) = 1/4 (exact).
constexpr float kHadamardNorm = 0.25f;

__device__ __forceinline__ void hadamard16(float (&v)[16]) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1)
#pragma unroll
    for (int i = 0; i < 16; i += 2 * h)
#pragma unroll
      for (int j = i; j < i + h; ++j) {
        const float a = v[j], b = v[j + h];
        v[j] = __fadd_rn(a, b);
        v[j + h] = __fsub_rn(a, b);
      }
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(v[i], kHadamardNorm);
}

// ------------------------------------------- activation fused into the codes
// SegQuant (Spanish technical summary 1 and 2.B; Korean technical summary
// section 2 "DualScale"): the small negative tail DualScale keeps comes from
// the SiLU / GELU that produces the layer input.  The fused producer reads
// the pre-activation z and quantizes x = act(z) without storing x:
//   SiLU(z) = z / (1 + e^-z),  GELU(z) = z/2 * erfc(-z / sqrt 2) (the exact,
//   erf-based GELU),
// with x the exact value rounded once, to nearest even, to bf16 (the
// activation storage type of the workloads this replaces).
//
// Evaluation: in fp32 with CUDA's expf / erfcf, whose documented maximum
// errors (2 and 4 units in the last place) bound the fp32 result's relative
// error by `rel` units of 2^-24 (SiLU: the exponential, the sum and the
// quotient; GELU: erfcf, the rounded argument -- whose relative error 2^-23 is
// amplified by |d ln erfc(a) / d ln a| <= 2a^2 + 1 -- and two products), with a
// safety factor of about two.  When no bf16 rounding midpoint lies within that
// bound of the fp32 result, rounding it to bf16 gives the rounding of the
// exact value; otherwise (about one element in ten thousand) the activation
// is recomputed in fp64 (CUDA's exp / erfc, a relative error below 2^-44
// here) and rounded from there; so are results below 2^-110, where the fp32
// intermediates overflow or lose precision.
constexpr int ACT_SILU = 1, ACT_GELU = 2;

// bf16 round-to-nearest-even of a double, directly (no intermediate fp32
// rounding): the two bf16 neighbours of d and their midpoint are exact in
// double.
__device__ __forceinline__ float bf16_rn_of_double(double d) {
  const float f = __double2float_rz(d);                 // |f| <= |d|, same sign
  const uint32_t t = __float_as_uint(f) & 0xFFFF0000u;  // bf16 toward zero
  const float lo = __uint_as_float(t);
  const float hi = __uint_as_float(t + 0x10000u);       // next bf16 away from zero
  const double mid = 0.5 * ((double)lo + (double)hi);
  const double a = fabs(d), am = fabs(mid);
  if (a > am) return hi;
  if (a < am) return lo;
  return ((t >> 16) & 1u) ? hi : lo;                    // a tie goes to the even one
}

template <int ACT>
__device__ __forceinline__ double act_f64(float z) {
  const double zd = (double)z;
  if constexpr (ACT == ACT_SILU) return zd / (1.0 + exp(-zd));
  else return 0.5 * zd * erfc(-zd * 0.70710678118654752440);
}

template <int ACT>
__device__ __forceinline__ float act_bf16(float z) {
  float v, rel;
  if constexpr (ACT == ACT_SILU) {
    v = __fdiv_rn(z, __fadd_rn(1.0f, expf(-z)));
    rel = 16.0f;
  } else {
    const float a = __fmul_rn(z, -0.70710678f);
    v = __fmul_rn(__fmul_rn(0.5f, z), erfcf(a));
    rel = fmaf(8.0f * a, a, 24.0f);
  }
  // the bf16 rounding midpoint between v's two bf16 neighbours (same binade
  // as v, so v - mid is exact)
  const float mid = __uint_as_float((__float_as_uint(v) & 0xFFFF0000u) | 0x8000u);
  const float margin = rel * 5.9604645e-8f * fabsf(v);
  // Results below 2^-110 come from an exponential that overflowed (SiLU,
  // z < -87) or an erfc near or in the fp32 subnormal range (GELU, z < -12),
  // where the relative bound does not hold: those, like non-finite results,
  // take the fp64 path too.
  if (fabsf(__fsub_rn(v, mid)) <= margin || !(fabsf(v) >= 0x1p-110f) ||
      !(fabsf(v) <= 3.4028234663852886e38f))
    return bf16_rn_of_double(act_f64<ACT>(z));
  return __bfloat162float(__float2bfloat16_rn(v));
}

template <int ACT>
__device__ __forceinline__ void act16(float (&v)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = act_bf16<ACT>(v[i]);
}

// blockDim = (32, 8): lane x owns the 16-element group blockIdx.x*32 + x of
// every row it visits (rows blockIdx.y*8 + y, stepping by gridDim.y*8), so its
// segment and reciprocal scales are fixed; a warp reads 1 KiB (bf16) and
// writes 512 bytes of each code tensor per row.
// MODE: CODES_DUAL (q+ and q-), CODES_COMBINED (c = q+ + q-), CODES_SINGLE
// (the single-scale code: both branches with s = max(s+, s-)), CODES_HADAMARD
// (q+ and q- of the block-Hadamard-transformed activations).
// CODES_SILU / CODES_GELU: the combined code c of x = bf16_RN(act(z)) from the
// pre-activation z (the activation fused into the producer).
constexpr int CODES_DUAL = 0, CODES_COMBINED = 1, CODES_SINGLE = 2, CODES_HADAMARD = 3,
              CODES_SILU = 4, CODES_GELU = 5;

template <typename XT, int MODE>
__device__ __forceinline__ void quantize_activations_body(
    const XT* __restrict__ x, int32_t M, int32_t K, int64_t ldx, SegBounds kseg,
    const float* __restrict__ s_pos, const float* __restrict__ s_neg, int8_t* __restrict__ q_pos,
    int8_t* __restrict__ q_neg, int64_t ldq) {
  const int32_t k = (blockIdx.x * 32 + threadIdx.x) * 16;
  if (k >= K) return;
  const int j = kseg.segment_of(k);
  constexpr bool COMBINED = (MODE == CODES_COMBINED || MODE == CODES_SINGLE ||
                            MODE == CODES_SILU || MODE == CODES_GELU);
  const float sj_p = (MODE == CODES_SINGLE) ? fmaxf(s_pos[j], s_neg[j]) : s_pos[j];
  const float sj_n = (MODE == CODES_SINGLE) ? sj_p : s_neg[j];
  const float rp = sj_p > 0.0f ? __frcp_rn(sj_p) : 0.0f;
  const float rn = sj_n > 0.0f ? __frcp_rn(sj_n) : 0.0f;
  const int32_t step = gridDim.y * 8;
  for (int32_t m = blockIdx.y * 8 + threadIdx.y; m < M; m += step) {
    float v[16];
    load16<XT>(x + (int64_t)m * ldx + k, v);
    if constexpr (MODE == CODES_HADAMARD) hadamard16(v);
    if constexpr (MODE == CODES_SILU) act16<ACT_SILU>(v);
    if constexpr (MODE == CODES_GELU) act16<ACT_GELU>(v);
    uint32_t p[16], n[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) { p[i] = code_pos(v[i], rp); n[i] = code_neg(v[i], rn); }
    if constexpr (COMBINED) {
#pragma unroll
      for (int i = 0; i < 16; ++i) p[i] += n[i];
    }
    uint4 up;
    up.x = pack4_low(p[0], p[1], p[2], p[3]);   up.y = pack4_low(p[4], p[5], p[6], p[7]);
    up.z = pack4_low(p[8], p[9], p[10], p[11]); up.w = pack4_low(p[12], p[13], p[14], p[15]);
    *reinterpret_cast<uint4*>(q_pos + (int64_t)m * ldq + k) = up;
    if constexpr (!COMBINED) {
      uint4 un;
      un.x = pack4_low(n[0], n[1], n[2], n[3]);   un.y = pack4_low(n[4], n[5], n[6], n[7]);
      un.z = pack4_low(n[8], n[9], n[10], n[11]); un.w = pack4_low(n[12], n[13], n[14], n[15]);
      *reinterpret_cast<uint4*>(q_neg + (int64_t)m * ldq + k) = un;
    }
  }
}

template <typename XT>
__global__ void __launch_bounds__(256) quantize_activations_kernel(
    const XT* __restrict__ x, int32_t M, int32_t K, int64_t ldx, SegBounds kseg,
    const float* __restrict__ s_pos, const float* __restrict__ s_neg, int8_t* __restrict__ q_pos,
    int8_t* __restrict__ q_neg, int64_t ldq) {
  quantize_activations_body<XT, CODES_DUAL>(x, M, K, ldx, kseg, s_pos, s_neg, q_pos, q_neg, ldq);
}

template <typename XT>
__global__ void __launch_bounds__(256) quantize_activations_hadamard_kernel(
    const XT* __restrict__ x, int32_t M, int32_t K, int64_t ldx, SegBounds kseg,
    const float* __restrict__ s_pos, const float* __restrict__ s_neg, int8_t* __restrict__ q_pos,
    int8_t* __restrict__ q_neg, int64_t ldq) {
  quantize_activations_body<XT, CODES_HADAMARD>(x, M, K, ldx, kseg, s_pos, s_neg, q_pos, q_neg, ldq);
}

// ------------------------------------------ table-driven activation (bf16 Z)
// A bf16 pre-activation has 65536 possible bit patterns, so x = act(z) for bf16
// z is a table: lut[b] = bits of bf16_RN(act(z_b)), filled by act_table_kernel
// with act_bf16 itself (the same values the direct path computes); non-finite
// patterns map to a quiet NaN (inputs must be finite).
constexpr int kActTableSize = 65536;

template <int ACT>
__global__ void __launch_bounds__(256) act_table_kernel(uint16_t* __restrict__ lut) {
  const int b = blockIdx.x * 256 + threadIdx.x;
  const float z = __uint_as_float((uint32_t)b << 16);
  uint16_t r = 0x7FC0u;
  if (fabsf(z) <= 3.4028234663852886e38f) r = (uint16_t)(__float_as_uint(act_bf16<ACT>(z)) >> 16);
  lut[b] = r;
}

// Combined codes of x = act(z) for bf16 z through the table, staged in shared
// memory (128 KiB, one block of 1024 threads per SM).  blockDim = (32, 32):
// lane x owns the 16-element group blockIdx.x*32 + x of every row it visits
// (rows blockIdx.y*32 + y, stepping by gridDim.y*32, two rows per iteration
// so that four 16-byte loads are in flight per thread); the reciprocal scales
// of every segment sit in shared memory.
constexpr int kActRowsPerIter = 2;

__global__ void __launch_bounds__(1024, 1) quantize_combined_act_table_kernel(
    const __nv_bfloat16* __restrict__ z, int32_t M, int32_t K, int64_t ldz, SegBounds kseg,
    const float* __restrict__ s_pos, const float* __restrict__ s_neg,
    const uint16_t* __restrict__ lut, int8_t* __restrict__ c, int64_t ldc) {
  extern __shared__ __align__(16) uint16_t tab[];     // kActTableSize entries
  __shared__ float sh_rp[SQ_MAX_SEG], sh_rn[SQ_MAX_SEG];
  const int tid = threadIdx.y * 32 + threadIdx.x;
  {
    const uint4* src = reinterpret_cast<const uint4*>(lut);
    uint4* dst = reinterpret_cast<uint4*>(tab);
    for (int i = tid; i < kActTableSize * 2 / 16; i += 1024) dst[i] = __ldg(src + i);
  }
  if (tid < kseg.count) {
    const float sp = s_pos[tid], sn = s_neg[tid];
    sh_rp[tid] = sp > 0.0f ? __frcp_rn(sp) : 0.0f;
    sh_rn[tid] = sn > 0.0f ? __frcp_rn(sn) : 0.0f;
  }
  __syncthreads();
  const int32_t k = (blockIdx.x * 32 + threadIdx.x) * 16;
  if (k >= K) return;
  const int j = kseg.segment_of(k);
  const float rp = sh_rp[j], rn = sh_rn[j];
  const int32_t step = gridDim.y * 32;
  auto codes16 = [&](const uint4 (&u)[2], uint4& out) {
    uint32_t p[16];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t w[4] = {u[h].x, u[h].y, u[h].z, u[h].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float x0 = __uint_as_float((uint32_t)tab[w[i] & 0xFFFFu] << 16);
        const float x1 = __uint_as_float((uint32_t)tab[w[i] >> 16] << 16);
        p[8 * h + 2 * i] = code_pos(x0, rp) + code_neg(x0, rn);
        p[8 * h + 2 * i + 1] = code_pos(x1, rp) + code_neg(x1, rn);
      }
    }
    out.x = pack4_low(p[0], p[1], p[2], p[3]);   out.y = pack4_low(p[4], p[5], p[6], p[7]);
    out.z = pack4_low(p[8], p[9], p[10], p[11]); out.w = pack4_low(p[12], p[13], p[14], p[15]);
  };
  int32_t m = blockIdx.y * 32 + threadIdx.y;
  for (; m + step < M; m += kActRowsPerIter * step) {
    uint4 u[kActRowsPerIter][2];
#pragma unroll
    for (int r = 0; r < kActRowsPerIter; ++r) {
      const uint4* src = reinterpret_cast<const uint4*>(z + (int64_t)(m + r * step) * ldz + k);
      u[r][0] = __ldg(src);
      u[r][1] = __ldg(src + 1);
    }
#pragma unroll
    for (int r = 0; r < kActRowsPerIter; ++r) {
      uint4 o;
      codes16(u[r], o);
      *reinterpret_cast<uint4*>(c + (int64_t)(m + r * step) * ldc + k) = o;
    }
  }
  if (m < M) {
    uint4 u[2];
    const uint4* src = reinterpret_cast<const uint4*>(z + (int64_t)m * ldz + k);
    u[0] = __ldg(src);
    u[1] = __ldg(src + 1);
    uint4 o;
    codes16(u, o);
    *reinterpret_cast<uint4*>(c + (int64_t)m * ldc + k) = o;
  }
}

// Calibration of transformed activations: per K segment max(T+) / 127 and
// max(-T-) / 127 of T = XH (XF = CODES_HADAMARD) or T = bf16_RN(act(Z))
// (XF = CODES_SILU / CODES_GELU, Z the pre-activation).  blockDim = (32, 8)
// with the quantizer's layout (lane x owns the 16-element group
// blockIdx.x*32 + x of every row it visits); eight lanes cover 128 columns,
// which never straddle a segment bound, so an eight-lane shuffle reduction is
// exact; then shared and global atomicMax on the fp32 bit patterns as in
// calibrate_kernel.  The outputs must be zeroed before the launch.
template <typename XT, int XF = CODES_HADAMARD>
__global__ void __launch_bounds__(256) calibrate_transformed_kernel(const XT* __restrict__ x,
                                                                 int64_t rows, int32_t K,
                                                                 int64_t ldx, SegBounds kseg,
                                                                 float* __restrict__ s_pos,
                                                                 float* __restrict__ s_neg) {
  __shared__ unsigned int sh_p[SQ_MAX_SEG], sh_n[SQ_MAX_SEG];
  __shared__ int sh_bad;
  const int tid = threadIdx.y * 32 + threadIdx.x;
  if (tid < SQ_MAX_SEG) { sh_p[tid] = 0u; sh_n[tid] = 0u; }
  if (tid == 0) sh_bad = 0;
  __syncthreads();
  const int32_t k = (blockIdx.x * 32 + threadIdx.x) * 16;
  const bool active = k < K;
  const int j = active ? kseg.segment_of(k) : 0;
  float P = 0.0f, Q = 0.0f;
  bool bad = false;
  if (active) {
    const int64_t step = (int64_t)gridDim.y * 8;
    for (int64_t m = (int64_t)blockIdx.y * 8 + threadIdx.y; m < rows; m += step) {
      float v[16];
      load16<XT>(x + m * ldx + k, v);
      if constexpr (XF == CODES_HADAMARD) hadamard16(v);
      if constexpr (XF == CODES_SILU) act16<ACT_SILU>(v);
      if constexpr (XF == CODES_GELU) act16<ACT_GELU>(v);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        bad |= (v[i] != v[i]) || (fabsf(v[i]) == __int_as_float(0x7f800000));
        P = fmaxf(P, v[i]);
        Q = fmaxf(Q, -v[i]);
      }
    }
  }
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) {
    P = fmaxf(P, __shfl_xor_sync(0xffffffffu, P, o));
    Q = fmaxf(Q, __shfl_xor_sync(0xffffffffu, Q, o));
  }
  const unsigned any_bad = __ballot_sync(0xffffffffu, bad);
  if (active && (threadIdx.x & 7) == 0) {
    atomicMax(&sh_p[j], __float_as_uint(P));
    atomicMax(&sh_n[j], __float_as_uint(Q));
  }
  if (threadIdx.x == 0 && any_bad) sh_bad = 1;
  __syncthreads();
  if (tid < kseg.count) {
    const float p = __uint_as_float(sh_p[tid]) / 127.0f;
    const float q = __uint_as_float(sh_n[tid]) / 127.0f;
    if (p > 0.0f) atomicMax(reinterpret_cast<unsigned int*>(s_pos) + tid, __float_as_uint(p));
    if (q > 0.0f) atomicMax(reinterpret_cast<unsigned int*>(s_neg) + tid, __float_as_uint(q));
  }
  if (tid == 0 && sh_bad) raise_status(SQ_STATUS_RANGE);
}

// Untransformed int4 weight codes rotated into the transform's basis: each
// 16-wide block of a row times the +-1 Sylvester matrix (exact integers; codes
// in [-7, 7] give values in [-112, 112]), written as int8.  One thread per
// (row, block): 8 packed bytes in (low nibble = even k), 16 bytes out.
__global__ void __launch_bounds__(256) rotate_weights_hadamard_kernel(
    const uint8_t* __restrict__ packed, int64_t N, int64_t K, int8_t* __restrict__ out,
    int64_t ldo) {
  const int64_t blocks = K / 16;
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= N * blocks) return;
  const int64_t n = t / blocks, b = t % blocks;
  const uint2 pk = __ldg(reinterpret_cast<const uint2*>(packed + n * (K / 2) + b * 8));
  const uint32_t w[2] = {pk.x, pk.y};
  int v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int nib = (int)((w[i >> 3] >> (4 * (i & 7))) & 0xFu);
    v[i] = (nib ^ 8) - 8;
  }
#pragma unroll
  for (int h = 1; h < 16; h <<= 1)
#pragma unroll
    for (int i = 0; i < 16; i += 2 * h)
#pragma unroll
      for (int jj = i; jj < i + h; ++jj) {
        const int a = v[jj], c = v[jj + h];
        v[jj] = a + c;
        v[jj + h] = a - c;
      }
  uint32_t o[4];
#pragma unroll
  for (int q = 0; q < 4; ++q)
    o[q] = (uint32_t)(v[4 * q] & 0xFF) | ((uint32_t)(v[4 * q + 1] & 0xFF) << 8) |
           ((uint32_t)(v[4 * q + 2] & 0xFF) << 16) | ((uint32_t)(v[4 * q + 3] & 0xFF) << 24);
  *reinterpret_cast<uint4*>(out + n * ldo + b * 16) = make_uint4(o[0], o[1], o[2], o[3]);
}

// Combined codes c = q+ + q- (one signed byte per activation): an element
// falls in exactly one branch, so the two magic-rounded words carry its code
// in their low bytes and the other branch's low byte is 0; their sum's low
// byte is c.  With MODE == CODES_SINGLE both branches use s = max(s+, s-), and
// c is the single-scale symmetric code.
template <typename XT, int MODE>
__global__ void __launch_bounds__(256) quantize_activations_combined_kernel(
    const XT* __restrict__ x, int32_t M, int32_t K, int64_t ldx, SegBounds kseg,
    const float* __restrict__ s_pos, const float* __restrict__ s_neg, int8_t* __restrict__ c,
    int64_t ldc) {
  quantize_activations_body<XT, MODE>(x, M, K, ldx, kseg, s_pos, s_neg, c, nullptr, ldc);
}

// ------------------------------------------------------ weight quantization
// int8: one 128-thread block per (output channel n, K segment j).  Pass 1:
// |W| max (warp shuffles, then shared memory); s = max/127; r = 1/s.  Pass 2
// (the segment row is now in L1): codes with the same magic rounding, clamp
// to +-127, sixteen codes per 16-byte store (segment bounds are multiples of
// 128 and K of 16).
template <typename WT>
__global__ void __launch_bounds__(128) quantize_weights_w8_kernel(
    const WT* __restrict__ w, int64_t N, int64_t K, int64_t ldw, SegBounds kseg,
    int8_t* __restrict__ codes, float* __restrict__ scales) {
  __shared__ float sh_max[4];
  __shared__ int sh_bad;
  const int64_t n = blockIdx.x / kseg.count;
  const int j = (int)(blockIdx.x - n * kseg.count);
  const int32_t k0 = kseg.b[j], k1 = kseg.b[j + 1];
  const WT* row = w + n * ldw;
  const int tid = threadIdx.x, lane = tid & 31;
  if (tid == 0) sh_bad = 0;
  // A segment row of up to 128 x 16 x 2 values stays in registers between the
  // two passes (both loads in flight at once, one read of the row).
  constexpr int kRegIters = 2;
  const bool in_regs = (k1 - k0) <= 128 * 16 * kRegIters;
  float vr[kRegIters][16];
  float amax = 0.0f;
  bool bad = false;
  if (in_regs) {
#pragma unroll
    for (int it = 0; it < kRegIters; ++it)
      if (k0 + tid * 16 + it * 128 * 16 < k1) load16<WT>(row + k0 + tid * 16 + it * 128 * 16, vr[it]);
#pragma unroll
    for (int it = 0; it < kRegIters; ++it)
      if (k0 + tid * 16 + it * 128 * 16 < k1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float a = fabsf(vr[it][i]);
          bad |= !(a <= 3.4028234663852886e38f);
          amax = fmaxf(amax, a);
        }
      }
  } else {
    for (int32_t k = k0 + tid * 16; k < k1; k += 128 * 16) {
      float v[16];
      load16<WT>(row + k, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float a = fabsf(v[i]);
        bad |= !(a <= 3.4028234663852886e38f);
        amax = fmaxf(amax, a);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const bool wbad = __any_sync(0xffffffffu, bad);
  __syncthreads();
  if (lane == 0) {
    sh_max[tid >> 5] = amax;
    if (wbad) sh_bad = 1;
  }
  __syncthreads();
  amax = fmaxf(fmaxf(sh_max[0], sh_max[1]), fmaxf(sh_max[2], sh_max[3]));
  if (tid == 0 && sh_bad) raise_status(SQ_STATUS_RANGE);
  const float s = amax / 127.0f;
  const float r = s > 0.0f ? __frcp_rn(s) : 0.0f;
  if (tid == 0) scales[(int64_t)j * N + n] = s;
  auto store16 = [&](const float (&v)[16], int32_t k) {
    uint32_t c[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      c[i] = __float_as_uint(fminf(fmaxf(fmaf(v[i], r, kMagic), kMagic - 127.0f), kMagic + 127.0f));
    uint4 out;
    out.x = pack4_low(c[0], c[1], c[2], c[3]);   out.y = pack4_low(c[4], c[5], c[6], c[7]);
    out.z = pack4_low(c[8], c[9], c[10], c[11]); out.w = pack4_low(c[12], c[13], c[14], c[15]);
    *reinterpret_cast<uint4*>(codes + n * K + k) = out;
  };
  if (in_regs) {
#pragma unroll
    for (int it = 0; it < kRegIters; ++it) {
      const int32_t k = k0 + tid * 16 + it * 128 * 16;
      if (k < k1) store16(vr[it], k);
    }
    return;
  }
  for (int32_t k = k0 + tid * 16; k < k1; k += 128 * 16) {
    float v[16];
    load16<WT>(row + k, v);
    store16(v, k);
  }
}

// int4: one warp per (output channel n, 128-wide group g); lane l owns k =
// 128g + 4l .. 4l+3.  s16 = fp16_rne(max/7) (fp32 division, then one RNE to
// binary16); codes use the widened fp16 scale; two codes per byte, low nibble
// = even k; scales stored group-major [K/128][N].
template <typename WT>
__global__ void __launch_bounds__(256) quantize_weights_w4_kernel(
    const WT* __restrict__ w, int64_t N, int64_t K, int64_t ldw, uint8_t* __restrict__ packed,
    __half* __restrict__ scales) {
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t G = K / 128;
  if (warp >= N * G) return;
  const int64_t n = warp / G;
  const int64_t g = warp - n * G;
  const WT* src = w + n * ldw + g * 128 + lane * 4;   // 16-byte (fp32) / 8-byte (bf16) aligned
  float v[4];
  if constexpr (sizeof(WT) == 4) {
    const float4 t = __ldg(reinterpret_cast<const float4*>(src));
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  } else {
    const uint2 t = __ldg(reinterpret_cast<const uint2*>(src));
    v[0] = __uint_as_float(t.x << 16); v[1] = __uint_as_float(t.x & 0xFFFF0000u);
    v[2] = __uint_as_float(t.y << 16); v[3] = __uint_as_float(t.y & 0xFFFF0000u);
  }
  float amax = 0.0f;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = fabsf(v[i]);
    bad |= !(a <= 3.4028234663852886e38f);
    amax = fmaxf(amax, a);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const __half s16 = __float2half_rn(amax / 7.0f);
  const float sf = __half2float(s16);
  bad |= !(sf <= 65504.0f);
  if (__any_sync(0xffffffffu, bad) && lane == 0) raise_status(SQ_STATUS_RANGE);
  const float r = sf > 0.0f ? __frcp_rn(sf) : 0.0f;
  uint32_t q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float t = fmaf(v[i], r, kMagic);
    t = fminf(fmaxf(t, kMagic - 7.0f), kMagic + 7.0f);
    q[i] = __float_as_uint(t) & 0xFu;  // two's complement nibble
  }
  const uint16_t two = (uint16_t)(q[0] | (q[1] << 4) | (q[2] << 8) | (q[3] << 12));
  *reinterpret_cast<uint16_t*>(packed + n * (K / 2) + g * 64 + lane * 2) = two;
  if (lane == 0) scales[g * N + n] = s16;
}

}  // namespace sq
