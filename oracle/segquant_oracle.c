/*
 * SegQuant DualScale / SegLinear quantized linear -- CPU ORACLE.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * statement of what the quantized linear layer computes.  It exists so that
 * the CUDA path can be checked against it.  Only the test suite, the smoke
 * check and the benchmark's CPU-baseline leg may load it.  It shares no code,
 * header, table or constant with the CUDA library, and the CUDA library never
 * calls it.
 *
 * Sources (gist.science summaries of "SegQuant: A Semantics-Aware and
 * Generalizable Quantization Framework for Diffusion Models"):
 *   [ES 2.B]  Spanish technical summary, section 2.B "DualScale": the
 *             activation X is split into its non-negative part X+ and its
 *             negative part X-, each with its own scale (s+, s-); the two
 *             products are computed as separate matrix multiplications and
 *             combined in the epilogue.
 *   [ES 2.A]  same page, section 2.A "SegLinear": input segments coming from
 *             a concatenation are quantized per semantic branch; output
 *             segments of a chunked output are quantized independently.
 *   [KO 2.2]  Korean technical summary, section 2 "DualScale": same split,
 *             "non-negative" region goes with s+.
 *   [KO 2.1]  Korean technical summary, section 2 "SegLinear": each segment
 *             gets an independent quantization scale.
 * The pages give no constants.  The workload specification of this project
 * fixes: s = max/127 per polarity, round-half-to-even, clamp +-127, symmetric
 * per-output-channel int8 weights, int4 weights in [-7,7] with group 128 and an
 * fp16 scale per group, two codes per byte.  Where both are silent this file
 * takes the readings R1..R9 listed next to each function.
 *
 * Precision: integer codes are decided in fp32 (the precision the scales are
 * defined in); accumulators are exact integers; the epilogue is evaluated in
 * fp32 in one fixed order (R9), so that the expected output is a single,
 * reproducible fp32 value.  The tests pin this fp32 evaluation to the exact
 * rational value of the definition within a derived rounding bound.
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -shared -fPIC (no fast-math; the
 * default rounding mode, round-to-nearest-even, is assumed throughout).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SQO_OK 0
#define SQO_ERR_ARG 1
#define SQO_ERR_RANGE 4

/* ---- element access ----------------------------------------------------- */

/* dtype 0: IEEE fp32; dtype 1: bfloat16 stored as its 16-bit pattern.
 * Widening bf16 -> fp32 is exact: the bf16 pattern is the top half of the
 * fp32 pattern. */
static float load_elem(const void* base, int dtype, int64_t idx) {
  if (dtype == 0) return ((const float*)base)[idx];
  uint32_t u = (uint32_t)((const uint16_t*)base)[idx] << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* fp32 -> bf16, round to nearest, ties to even (NaN kept quiet). */
uint16_t sqo_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

/* fp32 -> IEEE binary16, round to nearest, ties to even, overflow -> inf.
 * Written from the binary16 format definition (1 sign, 5 exponent bits with
 * bias 15, 10 fraction bits, subnormals below 2^-14). */
uint16_t sqo_f32_to_f16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  uint32_t absu = u & 0x7fffffffu;
  if (absu > 0x7f800000u) return (uint16_t)(sign | 0x7e00u); /* NaN */
  if (absu == 0x7f800000u) return (uint16_t)(sign | 0x7c00u); /* inf */
  float a;
  memcpy(&a, &absu, 4);
  /* Work in double: a is exact there, and a * 2^24 is an exact scaling. */
  double d = (double)a;
  if (d >= 65520.0) return (uint16_t)(sign | 0x7c00u); /* rounds to inf */
  if (d < 6.103515625e-05) { /* below 2^-14: subnormal grid of 2^-24 */
    double q = nearbyint(d * 16777216.0); /* exact scaling, RNE */
    return (uint16_t)(sign | (uint16_t)q); /* q == 1024 gives the smallest normal */
  }
  int e;
  double m = frexp(d, &e); /* d = m * 2^e, m in [0.5, 1) */
  /* 11 significant bits: scale m to [1024, 2048). */
  double q = nearbyint(m * 2048.0);
  if (q == 2048.0) { q = 1024.0; e += 1; }
  int biased = e - 1 + 15; /* value = (q/1024) * 2^(e-1) */
  if (biased >= 31) return (uint16_t)(sign | 0x7c00u);
  return (uint16_t)(sign | (uint16_t)(biased << 10) | (uint16_t)((uint32_t)q - 1024u));
}

float sqo_f16_to_f32(uint16_t h) {
  uint32_t sign = (h >> 15) & 1u, ex = (h >> 10) & 0x1fu, fr = h & 0x3ffu;
  double v;
  if (ex == 0) v = ldexp((double)fr, -24);
  else if (ex == 31) v = fr ? NAN : INFINITY;
  else v = ldexp((double)(fr + 1024u), (int)ex - 25);
  return (float)(sign ? -v : v);
}

/* ---- R2: reciprocal of a scale ------------------------------------------- */
/* Reading: codes are formed by multiplying by r = 1/s computed once in fp32
 * (IEEE division); a zero scale gives r = 0 and therefore all-zero codes. */
static float recip(float s) { return s > 0.0f ? 1.0f / s : 0.0f; }

/* ---- R4: round half to even of the exact product, then clamp ------------- */
/* x and r are fp32 (24-bit significands), so (double)x * (double)r is the
 * exact real product (48 bits < 53).  nearbyint rounds half to even under the
 * default rounding mode.  Infinite products saturate at the clamp. */
static int32_t round_clamp(float x, float r, int32_t lo, int32_t hi) {
  if (r == 0.0f || x == 0.0f) return 0;
  double p = nearbyint((double)x * (double)r);
  if (p < (double)lo) return lo;
  if (p > (double)hi) return hi;
  return (int32_t)p;
}

/* ---- R1: static calibration ------------------------------------------------
 * [ES 2.B], [KO 2.2]: one scale per polarity.  [ES 2.A], [KO 2.1]: one set of
 * scales per input (K) segment.  Workload specification: s+ = max(X+)/127,
 * s- = max(|X-|)/127, fp32 division.
 * x: rows x K with row stride ldx (elements); kb: J+1 segment bounds.
 * Returns SQO_ERR_RANGE if any input is NaN or a maximum is infinite. */
int sqo_calibrate(const void* x, int dtype, int64_t rows, int64_t K, int64_t ldx,
                  int32_t J, const int32_t* kb, float* s_pos, float* s_neg) {
  if (J < 1 || kb[0] != 0 || kb[J] != K) return SQO_ERR_ARG;
  int bad = 0;
  for (int32_t j = 0; j < J; ++j) {
    float P = 0.0f, Q = 0.0f;
    for (int64_t m = 0; m < rows; ++m) {
      for (int64_t k = kb[j]; k < kb[j + 1]; ++k) {
        float v = load_elem(x, dtype, m * ldx + k);
        if (v != v) bad = 1;
        if (v > P) P = v;
        if (-v > Q) Q = -v;
      }
    }
    s_pos[j] = P / 127.0f;
    s_neg[j] = Q / 127.0f;
    if (isinf(P) || isinf(Q)) bad = 1;
  }
  return bad ? SQO_ERR_RANGE : SQO_OK;
}

/* ---- R3/R4: DualScale activation codes ----------------------------------------
 * [ES 2.B], [KO 2.2]: X = X+ + X-; a non-negative element (including -0.0,
 * which compares equal to zero) belongs to X+, a negative one to X-; the other
 * branch holds 0 for that element.
 * q+ = clamp(RNE(x * r+), 0, 127), q- = clamp(RNE(x * r-), -127, 0). */
int sqo_quantize_activations(const void* x, int dtype, int64_t M, int64_t K, int64_t ldx,
                             int32_t J, const int32_t* kb, const float* s_pos,
                             const float* s_neg, int8_t* q_pos, int8_t* q_neg) {
  if (J < 1 || kb[0] != 0 || kb[J] != K) return SQO_ERR_ARG;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int32_t j = 0; j < J; ++j) {
      float rp = recip(s_pos[j]), rn = recip(s_neg[j]);
      for (int64_t k = kb[j]; k < kb[j + 1]; ++k) {
        float v = load_elem(x, dtype, m * ldx + k);
        int32_t qp = 0, qn = 0;
        if (v >= 0.0f) qp = round_clamp(v, rp, 0, 127);
        else if (v < 0.0f) qn = round_clamp(v, rn, -127, 0);
        q_pos[m * K + k] = (int8_t)qp;
        q_neg[m * K + k] = (int8_t)qn;
      }
    }
  }
  return SQO_OK;
}

/* ---- R5: int8 weights, symmetric, per output channel and per K segment -------
 * Workload specification: symmetric per-output-channel int8.  [ES 2.A]
 * ("quantize each semantic branch separately") read as: one scale per
 * (output channel n, input segment j).  With J = 1 this is plain per-channel.
 * s_w[j][n] = max_{k in seg j} |W[n,k]| / 127 (fp32);
 * q = clamp(RNE(w * (1/s_w)), -127, 127). */
int sqo_quantize_weights_w8(const float* w, int64_t N, int64_t K, int64_t ldw, int32_t J,
                            const int32_t* kb, int8_t* codes, float* scales) {
  if (J < 1 || kb[0] != 0 || kb[J] != K) return SQO_ERR_ARG;
  int bad = 0;
  for (int64_t n = 0; n < N; ++n) {
    for (int32_t j = 0; j < J; ++j) {
      float amax = 0.0f;
      for (int64_t k = kb[j]; k < kb[j + 1]; ++k) {
        float a = fabsf(w[n * ldw + k]);
        if (a != a || isinf(a)) bad = 1;
        if (a > amax) amax = a;
      }
      float s = amax / 127.0f;
      float r = recip(s);
      scales[(int64_t)j * N + n] = s;
      for (int64_t k = kb[j]; k < kb[j + 1]; ++k)
        codes[n * K + k] = (int8_t)round_clamp(w[n * ldw + k], r, -127, 127);
    }
  }
  return bad ? SQO_ERR_RANGE : SQO_OK;
}

/* ---- R6: int4 weights, group 128 along K, fp16 scale per group ----------------
 * Workload specification: symmetric int4 in [-7, 7], group size 128 along K,
 * two values per byte, one fp16 scale per group.  Readings: the group scale is
 * fp16_RNE(max|W|/7) with the division in fp32; codes use the fp16 scale
 * widened back to fp32; in each byte the low nibble holds the even k.
 * packed: [N][K/2] bytes; scales: [K/128][N] binary16 patterns (group-major). */
int sqo_quantize_weights_w4(const float* w, int64_t N, int64_t K, int64_t ldw, int32_t group,
                            uint8_t* packed, uint16_t* scales) {
  if (group != 128 || K % group != 0) return SQO_ERR_ARG;
  int64_t G = K / group;
  int bad = 0;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < G; ++g) {
      float amax = 0.0f;
      for (int64_t k = g * group; k < (g + 1) * group; ++k) {
        float a = fabsf(w[n * ldw + k]);
        if (a != a || isinf(a)) bad = 1;
        if (a > amax) amax = a;
      }
      uint16_t h = sqo_f32_to_f16(amax / 7.0f);
      if ((h & 0x7c00u) == 0x7c00u) bad = 1;
      scales[g * N + n] = h;
      float r = recip(sqo_f16_to_f32(h));
      for (int64_t k = g * group; k < (g + 1) * group; k += 2) {
        int32_t q0 = round_clamp(w[n * ldw + k], r, -7, 7);
        int32_t q1 = round_clamp(w[n * ldw + k + 1], r, -7, 7);
        packed[n * (K / 2) + k / 2] = (uint8_t)(((uint32_t)q0 & 0xfu) | (((uint32_t)q1 & 0xfu) << 4));
      }
    }
  }
  return bad ? SQO_ERR_RANGE : SQO_OK;
}

/* Unpack int4 codes to one int8 per element (sign extension of each nibble). */
void sqo_unpack_w4(const uint8_t* packed, int64_t N, int64_t K, int8_t* codes) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      uint8_t b = packed[n * (K / 2) + k / 2];
      int32_t v = (k & 1) ? (b >> 4) : (b & 0xf);
      if (v >= 8) v -= 16;
      codes[n * K + k] = (int8_t)v;
    }
}

/* ---- R8: the two integer GEMMs, one pair of accumulators per unit ------------
 * [ES 2.B], [KO 2.2]: X+^ W^ and X-^ W^ are computed as separate products.
 * A unit is a K segment (int8 weights) or a 128-wide K group (int4 weights);
 * ub holds U+1 unit bounds.  acc: [U][2][M][N] int32, polarity 0 = (+).
 * Sums are formed in int64 and must fit int32. */
int sqo_accumulate(const int8_t* q_pos, const int8_t* q_neg, int64_t M, int64_t K,
                   const int8_t* wcodes, int64_t N, int32_t U, const int32_t* ub,
                   int32_t* acc) {
  int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
  for (int64_t m = 0; m < M; ++m) {
    for (int32_t u = 0; u < U; ++u) {
      for (int64_t n = 0; n < N; ++n) {
        int64_t sp = 0, sn = 0;
        for (int64_t k = ub[u]; k < ub[u + 1]; ++k) {
          int64_t wv = wcodes[n * K + k];
          sp += (int64_t)q_pos[m * K + k] * wv;
          sn += (int64_t)q_neg[m * K + k] * wv;
        }
        if (sp > INT32_MAX || sp < INT32_MIN || sn > INT32_MAX || sn < INT32_MIN) bad = 1;
        acc[(((int64_t)u * 2 + 0) * M + m) * N + n] = (int32_t)sp;
        acc[(((int64_t)u * 2 + 1) * M + m) * N + n] = (int32_t)sn;
      }
    }
  }
  return bad ? SQO_ERR_RANGE : SQO_OK;
}

/* ---- R9: the fused epilogue ---------------------------------------------------
 * [ES 2.B] "combined in the epilogue"; [KO 2.2] "scaled results fused".
 * Workload specification: y = s_w[n] * (s+ * acc+ + s- * acc-) + bias.
 * Reading (fixed fp32 order): F = int32 -> fp32 (RNE);
 *   t_u = fmaf(s-_j, F(acc-_u), s+_j * F(acc+_u));
 *   y = 0; for u ascending: y = fmaf(sw_u[n], t_u, y);
 *   if bias: y = y + b[n];
 * unit_seg[u] = segment j of unit u; sw[u][n] = weight scale of unit u.
 * out_dtype 0: fp32 into y (float*), 1: bf16 patterns (uint16_t*). */
int sqo_epilogue(const int32_t* acc, int64_t M, int64_t N, int32_t U, const int32_t* unit_seg,
                 const float* s_pos, const float* s_neg, const float* sw, const float* bias,
                 void* y, int out_dtype, int64_t ldy) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t n = 0; n < N; ++n) {
      float acc_y = 0.0f;
      for (int32_t u = 0; u < U; ++u) {
        int32_t j = unit_seg[u];
        float fp = (float)acc[(((int64_t)u * 2 + 0) * M + m) * N + n];
        float fn = (float)acc[(((int64_t)u * 2 + 1) * M + m) * N + n];
        float prod = s_pos[j] * fp;
        float t = fmaf(s_neg[j], fn, prod);
        acc_y = fmaf(sw[(int64_t)u * N + n], t, acc_y);
      }
      if (bias) acc_y = acc_y + bias[n];
      if (out_dtype == 0) ((float*)y)[m * ldy + n] = acc_y;
      else ((uint16_t*)y)[m * ldy + n] = sqo_f32_to_bf16(acc_y);
    }
  }
  return SQO_OK;
}

/* ---- Single-scale baseline --------------------------------------------------
 * The summaries compare DualScale's latency with naive quantization [ES 4,
 * "Eficiencia y Despliegue"]; the naive scheme is the standard single-scale
 * quantization DualScale replaces [ES 2.B].  Reading: one symmetric scale per K
 * segment, s_j = max|x| / 127 over the calibration rows, which is
 * max(s+_j, s-_j) (fp32 division by 127 is monotone);
 * c = clamp(RNE(x * fl(1/s_j)), -127, 127); NaN -> 0 (as in the DualScale
 * codes, where NaN falls in neither branch). */
int sqo_quantize_activations_single(const void* x, int dtype, int64_t M, int64_t K, int64_t ldx,
                                    int32_t J, const int32_t* kb, const float* s_pos,
                                    const float* s_neg, int8_t* c) {
  if (J < 1 || kb[0] != 0 || kb[J] != K) return SQO_ERR_ARG;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int32_t j = 0; j < J; ++j) {
      float s = s_pos[j] > s_neg[j] ? s_pos[j] : s_neg[j];
      float r = recip(s);
      for (int64_t k = kb[j]; k < kb[j + 1]; ++k) {
        float v = load_elem(x, dtype, m * ldx + k);
        int32_t q = 0;
        if (v == v) q = round_clamp(v, r, -127, 127);
        c[m * K + k] = (int8_t)q;
      }
    }
  }
  return SQO_OK;
}

/* Single-scale epilogue (fixed fp32 order, the same shape as R9):
 *   t_u = s_j * F(acc_u); y = 0; for u ascending: y = fmaf(sw_u[n], t_u, y);
 *   if bias: y = y + b[n].
 * acc: int32 [U][M][N]. */
int sqo_epilogue_single(const int32_t* acc, int64_t M, int64_t N, int32_t U,
                        const int32_t* unit_seg, const float* s_pos, const float* s_neg,
                        const float* sw, const float* bias, void* y, int out_dtype, int64_t ldy) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t n = 0; n < N; ++n) {
      float acc_y = 0.0f;
      for (int32_t u = 0; u < U; ++u) {
        int32_t j = unit_seg[u];
        float s = s_pos[j] > s_neg[j] ? s_pos[j] : s_neg[j];
        float t = s * (float)acc[((int64_t)u * M + m) * N + n];
        acc_y = fmaf(sw[(int64_t)u * N + n], t, acc_y);
      }
      if (bias) acc_y = acc_y + bias[n];
      if (out_dtype == 0) ((float*)y)[m * ldy + n] = acc_y;
      else ((uint16_t*)y)[m * ldy + n] = sqo_f32_to_bf16(acc_y);
    }
  }
  return SQO_OK;
}

/* Keeps the fp32 value of the epilogue before any output rounding, for tests
 * that need the unrounded fp32 result (same order as sqo_epilogue). */
int sqo_epilogue_f32(const int32_t* acc, int64_t M, int64_t N, int32_t U,
                     const int32_t* unit_seg, const float* s_pos, const float* s_neg,
                     const float* sw, const float* bias, float* y) {
  return sqo_epilogue(acc, M, N, U, unit_seg, s_pos, s_neg, sw, bias, y, 0, N);
}

/* ---- Activation in front of the layer (the fused producer) -----------------
 * [ES 1], [ES 2.B], [KO 2.2]: the small negative tail DualScale keeps comes
 * from the SiLU / GELU that produces the layer input.  The fused producer
 * quantizes x = act(z) straight from the pre-activation z.
 *   act 1: SiLU(z) = z / (1 + exp(-z));
 *   act 2: GELU(z) = z/2 * erfc(-z / sqrt(2))  (the exact, erf-based GELU).
 * Reading: x is the exact act(z) rounded once, to nearest with ties to even,
 * to bf16.  Here act(z) is evaluated in double with the C library (relative
 * error far below 2^-40 for finite z); flags[i] = 1 when that double lies
 * within a relative 2^-40 of a bf16 rounding midpoint, where a library's error
 * could decide the rounding -- such elements are exempt from exact comparison.
 * z: fp32 or bf16 patterns (dtype as load_elem); x: bf16 patterns. */
static const double kBf16Max = 3.3895313892515355e38;   /* (2 - 2^-7) * 2^127 */

/* bf16 round-half-even of a double, from the format: 8 significant bits,
 * exponents down to -126, subnormal spacing 2^-133. */
static uint16_t bf16_from_double(double d, int* near_mid) {
  *near_mid = 0;
  const uint16_t sign = signbit(d) ? 0x8000u : 0u;
  double a = fabs(d);
  if (a == 0.0) return sign;
  int e;
  (void)frexp(a, &e);                 /* a in [2^(e-1), 2^e) */
  int E = e - 1;
  if (E < -126) E = -126;             /* subnormal range: fixed spacing */
  const double ulp = ldexp(1.0, E - 7);
  const double q = a / ulp;           /* exact: a power-of-two scaling */
  const double fl = floor(q);
  if (fabs(q - (fl + 0.5)) <= q * 0x1p-40) *near_mid = 1;
  const double r = nearbyint(q) * ulp;
  if (r > kBf16Max) return (uint16_t)(sign | 0x7f80u);   /* rounds to infinity */
  const float rf = (float)r;          /* exact: r has at most 8 significant bits */
  uint32_t u;
  memcpy(&u, &rf, 4);
  return (uint16_t)(sign | ((u >> 16) & 0x7fffu));
}

int sqo_activation_bf16(const void* z, int dtype, int64_t n, int act, uint16_t* x,
                        uint8_t* flags) {
  if (act != 1 && act != 2) return SQO_ERR_ARG;
  int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
  for (int64_t i = 0; i < n; ++i) {
    const double zd = (double)load_elem(z, dtype, i);
    if (!isfinite(zd)) bad = 1;
    const double v = (act == 1) ? zd / (1.0 + exp(-zd)) : 0.5 * zd * erfc(-zd / sqrt(2.0));
    int near_mid = 0;
    x[i] = bf16_from_double(v, &near_mid);
    flags[i] = (uint8_t)near_mid;
  }
  return bad ? SQO_ERR_RANGE : SQO_OK;
}
