/*
 * segquant.h -- C ABI of the B200 (sm_100a) DualScale / SegLinear quantized
 * linear layer.
 *
 * What the layer computes comes from the SegQuant summaries ("SegQuant: A
 * Semantics-Aware and Generalizable Quantization Framework for Diffusion
 * Models", gist.science):
 *   - DualScale (Spanish technical summary, section 2.B; Korean technical
 *     summary, section 2 "DualScale"): the activation X is split into its
 *     non-negative part X+ and its negative part X-, each quantized with its
 *     own static scale (s+, s-); the two integer products X+^ W^ and X-^ W^ run
 *     in one kernel and are combined in a fused epilogue.
 *   - SegLinear (Spanish technical summary, section 2.A; Korean technical
 *     summary, section 2 "SegLinear"): each input (K) segment of a linear
 *     layer has its own activation scales and its own weight scales; output (N)
 *     segments are quantized independently.
 *   - Static calibration (Spanish technical summary, section 1 "compiler gap";
 *     section 3 item 4): scales are fixed offline, no runtime-dynamic values.
 *
 * Numeric rules (every entry point follows them bit for bit):
 *   s+_j = max(max(x,0))/127, s-_j = max(max(-x,0))/127 over segment j (fp32
 *   division); r = 1/s in fp32 (0 when s = 0); a non-negative x (including
 *   -0.0) takes q+ = clamp(round_half_even(x*r+), 0, 127) and q- = 0; a
 *   negative x takes q- = clamp(round_half_even(x*r-), -127, 0) and q+ = 0,
 *   where x*r is the exact product.  int8 weights: s_w[j][n] =
 *   max_{k in seg j}|W[n,k]|/127, codes clamp(round_half_even(w/s), -127, 127).
 *   int4 weights: group 128 along K, s = fp16_rne(max|W|/7), codes in [-7, 7],
 *   two per byte, low nibble = even k.  Epilogue per output, for units u (a K
 *   segment for int8 weights, a 128-wide group for int4 weights) in ascending
 *   order: t = fmaf(s-_j, float(acc-_u), s+_j * float(acc+_u));
 *   y = fmaf(sw_u[n], t, y) starting from y = 0; then y += bias[n]; then the
 *   output conversion (fp32 as is, bf16 round-half-even).
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers owned by the caller unless marked "host".
 *     The library allocates no device memory and keeps no per-call state.
 *   - Matrices are row-major.  X is [M, K] (tokens x in-features, the
 *     nn.Linear input), W is [N, K] (the nn.Linear weight), Y is [M, N].
 *     Leading dimensions are in elements.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  Arguments are validated on the host before any
 *     launch; a rejected call enqueues nothing.  The GEMMs from codes are
 *     programmatic dependent launches: their setup may overlap the kernel
 *     before them in the stream, but they read their inputs and write Y only
 *     after that kernel has completed, so stream order holds as usual.
 *   - Device-side conditions (a non-finite calibration maximum, an fp16 group
 *     scale overflow, a bounded pipeline wait that expired) are recorded in a
 *     per-device status word and returned by sq_stream_status().
 *   - Inputs must be finite.  NaN activations, and an infinite activation whose
 *     polarity has a zero scale, produce unspecified codes.
 */
#ifndef SEGQUANT_H_
#define SEGQUANT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, spelled without the CUDA headers. */
typedef struct CUstream_st* sq_stream_t;

typedef enum {
  SQ_OK = 0,
  SQ_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad dtype, inconsistent sizes */
  SQ_ERR_ALIGNMENT = 2,   /* a pointer not 16-byte aligned or a row stride not a multiple of 16 bytes */
  SQ_ERR_UNSUPPORTED = 3, /* segment bound not a multiple of 128, N % 16 != 0, bits/group combination */
  SQ_ERR_RANGE = 4,       /* non-finite calibration maximum or weight, fp16 group scale overflow, size limit */
  SQ_ERR_CUDA = 5,        /* a CUDA runtime or driver call failed */
  SQ_ERR_TIMEOUT = 6      /* a bounded device-side pipeline wait expired (reported by sq_stream_status) */
} sq_status;

typedef enum { SQ_F32 = 0, SQ_BF16 = 1 } sq_dtype;

/* Largest number of K segments per layer, and the largest K. */
#define SQ_MAX_SEGMENTS 16
#define SQ_MAX_K 131072

/* Segment bounds, HOST memory: `count` segments, `count + 1` increasing bounds,
 * bounds[0] = 0 and bounds[count] = the extent (K or N).  K-segment bounds other
 * than the last must be multiples of 128. */
typedef struct {
  int32_t count;
  const int32_t* bounds;
} sq_segments;

/* A quantized weight.  The struct itself is host memory; `codes` and
 * `scales` are device buffers the caller allocates with the sizes returned by
 * sq_qweight_sizes().
 *   bits = 8, group = 0  : codes int8 [N][K]; scales fp32 [J][N] (J = kseg.count),
 *                          one scale per (K segment, output channel).
 *   bits = 4, group = 128: codes uint8 [N][K/2], low nibble = even k;
 *                          scales binary16 [K/128][N] (group-major), one per
 *                          (group, channel).
 * nseg (output segments, e.g. q | k | v) is validated and carried as metadata:
 * per-channel weight scales make an output split a numerical no-op. */
typedef struct {
  int32_t bits;
  int32_t group;
  int64_t N;
  int64_t K;
  sq_segments kseg;
  sq_segments nseg;
  void* codes;
  void* scales;
} sq_qweight;

/* Host only.  Byte sizes of the code and scale buffers of a quantized weight.
 * Errors: SQ_ERR_INVALID_ARG for null outputs or non-positive sizes,
 * SQ_ERR_UNSUPPORTED for a bits/group combination other than (8, 0), (4, 128)
 * or K % 128 != 0 with bits = 4. */
sq_status sq_qweight_sizes(int32_t bits, int64_t N, int64_t K, int32_t J, int32_t group,
                           size_t* code_bytes, size_t* scale_bytes);

/* Static DualScale calibration (SegQuant, Spanish technical summary 2.B and
 * 1 "compiler gap"; Korean technical summary section 2 "DualScale").
 * x: [rows, K] fp32 or bf16 with row stride ldx; the calibration rows.
 * kseg: host K-segment bounds.  s_pos, s_neg: device fp32 [J] outputs,
 * s+_j = max(x+)/127 and s-_j = max(|x-|)/127 over rows x segment j.
 * A NaN input or an infinite maximum sets SQ_ERR_RANGE in the status word.
 * rows = 0 gives zero scales.  Alignment: x 16-byte aligned, ldx*elt % 16 == 0. */
sq_status sq_calibrate(const void* x, sq_dtype xt, int64_t rows, int64_t K, int64_t ldx,
                       const sq_segments* kseg, float* s_pos, float* s_neg, sq_stream_t stream);

/* Weight quantization (SegQuant SegLinear: Spanish technical summary 2.A,
 * Korean technical summary section 2 "SegLinear"; int8 per channel and per K
 * segment, or int4 with group 128 and fp16 scales).
 * w: [N, K] fp32 or bf16 with row stride ldw.  `out` describes the
 * destination (bits, group, N, K, kseg, nseg, codes, scales preset by the
 * caller).  Non-finite weights or an fp16 scale overflow set SQ_ERR_RANGE in
 * the status word.  Alignment: w 16-byte aligned, ldw*elt % 16 == 0; codes and
 * scales 16-byte aligned. */
sq_status sq_quantize_weights(const void* w, sq_dtype wt, int64_t N, int64_t K, int64_t ldw,
                              const sq_qweight* out, sq_stream_t stream);

/* The fused forward pass: DualScale quantization of X inside the GEMM, the two
 * int8 tensor-core products per unit, the per-unit fold and the epilogue
 * (SegQuant, Spanish technical summary 2.B "BatchedGEMM ... fused in the
 * epilogue"; Korean technical summary section 2 "Fused Epilogue").
 * x: [M, K] fp32 or bf16, row stride ldx.  w: quantized weight (K must match).
 * s_pos, s_neg: device fp32 [J] activation scales.  bias: device fp32 [N] or
 * NULL.  y: [M, N] fp32 or bf16, row stride ldy.  M = 0 is a no-op.
 * Requirements: N % 16 == 0; K % 16 == 0 (K % 128 == 0 for int4 weights);
 * K <= SQ_MAX_K; x, y, codes, scales 16-byte aligned; ldx*elt and ldy*elt
 * multiples of 16 bytes. */
sq_status sq_linear_forward(const void* x, sq_dtype xt, int64_t M, int64_t K, int64_t ldx,
                            const sq_qweight* w, const float* s_pos, const float* s_neg,
                            const float* bias, void* y, sq_dtype yt, int64_t ldy,
                            sq_stream_t stream);

/* The forward pass from pre-quantized DualScale codes (the q+ / q- tensors
 * written by sq_quantize_activations with the same scales): the kernel loads
 * both int8 code tiles by TMA and runs the two tensor-core products and the
 * fused epilogue exactly as sq_linear_forward does, so the result is
 * identical.  Splitting quantization from the GEMM lets one quantization
 * serve every output tile instead of being redone per tile.
 * q_pos, q_neg: device int8 [M, K], row stride ldq (a multiple of 16), 16-byte
 * aligned.  Other arguments and requirements as for sq_linear_forward. */
sq_status sq_linear_forward_codes(const int8_t* q_pos, const int8_t* q_neg, int64_t ldq,
                                  int64_t M, int64_t K, const sq_qweight* w, const float* s_pos,
                                  const float* s_neg, const float* bias, void* y, sq_dtype yt,
                                  int64_t ldy, sq_stream_t stream);

/* Test / fallback surface: the DualScale codes alone (same rules as the
 * forward's in-kernel quantization).  q_pos, q_neg: device int8 [M, K] with row
 * stride ldq (a multiple of 16). */
sq_status sq_quantize_activations(const void* x, sq_dtype xt, int64_t M, int64_t K, int64_t ldx,
                                  const sq_segments* kseg, const float* s_pos,
                                  const float* s_neg, int8_t* q_pos, int8_t* q_neg, int64_t ldq,
                                  sq_stream_t stream);

/* DualScale codes in one byte per activation: c = q+ + q- (SegQuant DualScale,
 * Spanish technical summary 2.B: X = X+ + X-, the two parts have disjoint
 * support, so at most one of q+, q- is non-zero and c in [-127, 127] carries
 * both: q+ = max(c, 0), q- = min(c, 0)).  Same rules and scales as
 * sq_quantize_activations.  c: device int8 [M, K], row stride ldc (a multiple
 * of 16), 16-byte aligned; written by the call.  Requirements and errors as for
 * sq_quantize_activations. */
sq_status sq_quantize_activations_combined(const void* x, sq_dtype xt, int64_t M, int64_t K,
                                           int64_t ldx, const sq_segments* kseg,
                                           const float* s_pos, const float* s_neg, int8_t* c,
                                           int64_t ldc, sq_stream_t stream);

/* Activation fused into the combined-code producer.  SegQuant (Spanish
 * technical summary 1 and 2.B; Korean technical summary section 2,
 * "DualScale"): the negative tail DualScale preserves is produced by the SiLU /
 * GELU in front of the layer, so the producer reads the pre-activation Z and
 * writes the codes of X = act(Z) without storing X.
 *   SQ_ACT_SILU: act(z) = z / (1 + exp(-z));
 *   SQ_ACT_GELU: act(z) = z/2 * erfc(-z / sqrt(2)) (the exact, erf-based GELU).
 * Reading: x is the exact act(z) rounded once, to nearest even, to bf16 (the
 * storage type of the activations this replaces); the kernels evaluate it in
 * fp32 and fall back to fp64 wherever the fp32 error bound does not decide the
 * bf16 rounding, so x equals the correctly rounded value (up to fp64 ties). */
typedef enum { SQ_ACT_SILU = 1, SQ_ACT_GELU = 2 } sq_act;

/* Static DualScale scales of X = act(Z) over the calibration rows of Z (rows x
 * K, dtype zt, row stride ldz): sq_calibrate's rule applied to X.  Arguments,
 * requirements and errors as for sq_calibrate (K a multiple of 16); an
 * unknown `act` returns SQ_ERR_INVALID_ARG.  Z must be finite. */
sq_status sq_calibrate_act(const void* z, sq_dtype zt, sq_act act, int64_t rows, int64_t K,
                           int64_t ldz, const sq_segments* kseg, float* s_pos, float* s_neg,
                           sq_stream_t stream);

/* Combined DualScale codes c = q+ + q- of X = act(Z), read from the
 * pre-activation Z [M, K] (dtype zt, row stride ldz): one pass over Z, X never
 * written.  Codes, layout and requirements as for
 * sq_quantize_activations_combined; an unknown `act` returns
 * SQ_ERR_INVALID_ARG.  Z must be finite.  The codes feed
 * sq_linear_forward_combined. */
sq_status sq_quantize_activations_combined_act(const void* z, sq_dtype zt, sq_act act, int64_t M,
                                               int64_t K, int64_t ldz, const sq_segments* kseg,
                                               const float* s_pos, const float* s_neg, int8_t* c,
                                               int64_t ldc, sq_stream_t stream);

/* The forward pass from combined codes (written by
 * sq_quantize_activations_combined with the same scales): the kernel loads one
 * int8 code tile per k block by TMA, splits it into q+ and q- in shared memory
 * and runs the two tensor-core products and the fused epilogue of
 * sq_linear_forward, so the result is identical to sq_linear_forward and
 * sq_linear_forward_codes.  c: device int8 [M, K], row stride ldc (a multiple
 * of 16), 16-byte aligned.  int8 weights only (bits = 4 returns
 * SQ_ERR_UNSUPPORTED).  Other arguments and requirements as for
 * sq_linear_forward. */
sq_status sq_linear_forward_combined(const int8_t* c, int64_t ldc, int64_t M, int64_t K,
                                     const sq_qweight* w, const float* s_pos, const float* s_neg,
                                     const float* bias, void* y, sq_dtype yt, int64_t ldy,
                                     sq_stream_t stream);

/* Single-scale ("naive") baseline of the same layer, for the latency
 * comparison the SegQuant summaries make against naive quantization (Spanish
 * technical summary section 4, "Eficiencia y Despliegue"; the standard
 * single-scale quantization DualScale replaces, section 2.B).  Reading: one
 * symmetric scale per K segment, s_j = max|x| / 127 over the calibration rows,
 * which equals max(s_pos[j], s_neg[j]) from sq_calibrate (fp32 division by 127
 * is monotone); codes c = clamp(round_half_even(x * fl(1/s_j)), -127, 127),
 * NaN -> 0.  c: device int8 [M, K], row stride ldc (a multiple of 16),
 * 16-byte aligned.  Requirements and errors as for sq_quantize_activations. */
sq_status sq_quantize_activations_single(const void* x, sq_dtype xt, int64_t M, int64_t K,
                                         int64_t ldx, const sq_segments* kseg, const float* s_pos,
                                         const float* s_neg, int8_t* c, int64_t ldc,
                                         sq_stream_t stream);

/* The single-scale forward from codes written by sq_quantize_activations_single
 * with the same scales: one int8 tensor-core product per unit, epilogue (fixed
 * fp32 order) t = s_j * F(acc), y = fma(s_w[j][n], t, y) over the units from
 * y = 0, then + bias, then the output rounding.  int8 weights only (bits = 4
 * returns SQ_ERR_UNSUPPORTED).  Other arguments and requirements as for
 * sq_linear_forward_combined. */
sq_status sq_linear_forward_single(const int8_t* c, int64_t ldc, int64_t M, int64_t K,
                                   const sq_qweight* w, const float* s_pos, const float* s_neg,
                                   const float* bias, void* y, sq_dtype yt, int64_t ldy,
                                   sq_stream_t stream);

/* ---- Block-Hadamard activations (HQ-DM, "HQ-DM: Single Hadamard
 * Transformation-Based Quantization-Aware Training for Low-Bit Diffusion
 * Models", Spanish technical summary section 2.1): the activation matrix is
 * multiplied by a block-diagonal Hadamard matrix H before quantization, the
 * weights are quantized untransformed, and the activation is recovered as
 * X^ = S (XH)_int H (H orthogonal and symmetric), the block normalization
 * 2^(-k/2) carried by the floating-point scales.  Readings: blocks of 16 along
 * K (normalization 1/4); the transform in fp32 by the Sylvester-ordered
 * butterfly (stage h = 1, 2, 4, 8: (v[j], v[j+h]) -> (v[j] + v[j+h],
 * v[j] - v[j+h]), each rounded), then times 1/4; Y = X^ W^T evaluated exactly
 * as the integer product of the XH codes with the int4 weight codes rotated by
 * the +-1 Sylvester matrix, with the activation scales times 1/4 in the
 * DualScale epilogue.  int4 weights (group 128) only: their rotated codes lie
 * in [-112, 112] and stay int8. */

/* Per-segment DualScale scales of XH: s_pos[j] = max(XH+)/127, s_neg[j] =
 * max(-XH-)/127 over the rows (as sq_calibrate, on the transformed values).
 * K % 16 == 0; other arguments, requirements and errors as for sq_calibrate. */
sq_status sq_calibrate_hadamard(const void* x, sq_dtype xt, int64_t rows, int64_t K, int64_t ldx,
                                const sq_segments* kseg, float* s_pos, float* s_neg,
                                sq_stream_t stream);

/* DualScale codes of XH with the scales of sq_calibrate_hadamard (the codes of
 * sq_quantize_activations applied to the transformed row blocks).  Arguments,
 * requirements and errors as for sq_quantize_activations. */
sq_status sq_quantize_activations_hadamard(const void* x, sq_dtype xt, int64_t M, int64_t K,
                                           int64_t ldx, const sq_segments* kseg,
                                           const float* s_pos, const float* s_neg, int8_t* q_pos,
                                           int8_t* q_neg, int64_t ldq, sq_stream_t stream);

/* The int4 weight codes of w (bits = 4, group 128, as written by
 * sq_quantize_weights) rotated into the transform's basis: every 16-wide block
 * of a row times the +-1 Sylvester matrix, exact, written as int8.
 * w_rot: device int8 [N, K], row stride ldr (>= K, a multiple of 16), 16-byte
 * aligned, owned by the caller.  Errors: SQ_ERR_UNSUPPORTED for bits = 8;
 * SQ_ERR_INVALID_ARG / SQ_ERR_ALIGNMENT as for the other weight calls. */
sq_status sq_rotate_weights_hadamard(const sq_qweight* w, int8_t* w_rot, int64_t ldr,
                                     sq_stream_t stream);

/* The forward from the codes of sq_quantize_activations_hadamard: per 128-wide
 * group g, acc+- = q+- . w_rot^T (int32), then the DualScale epilogue with the
 * group's fp16 weight scale and the activation scales times 1/4:
 * t = fma(s-/4, F(acc-), (s+/4) * F(acc+)), y = fma(s_w[g][n], t, y), + bias,
 * output rounding.  w: the int4 weight the rotation was made from (its N, K,
 * K segments and group scales are used; its packed codes are not read);
 * w_rot, ldr: as written by sq_rotate_weights_hadamard.  s_pos/s_neg: the
 * scales of XH.  Other arguments and requirements as for
 * sq_linear_forward_codes; SQ_ERR_UNSUPPORTED for bits = 8. */
sq_status sq_linear_forward_codes_hadamard(const int8_t* q_pos, const int8_t* q_neg, int64_t ldq,
                                           int64_t M, int64_t K, const sq_qweight* w,
                                           const int8_t* w_rot, int64_t ldr, const float* s_pos,
                                           const float* s_neg, const float* bias, void* y,
                                           sq_dtype yt, int64_t ldy, sq_stream_t stream);

/* Small-M forward from DualScale codes (1 <= M <= 128 tokens): the same result
 * as sq_linear_forward_codes, bit for bit (SegQuant DualScale, Spanish
 * technical summary 2.B; the two int8 products and the fused epilogue), with
 * the weight stream spread over the whole GPU: the K dimension is split, each
 * (N tile, K split) unit computes int32 partial accumulators, and the last
 * unit of each output region adds them (integer sums are exact in any order)
 * and runs the epilogue.  Requirements beyond sq_linear_forward_codes: int8
 * weights with one K segment (else SQ_ERR_UNSUPPORTED); M <= 128 (else
 * SQ_ERR_UNSUPPORTED).
 * workspace: device memory, 256-byte aligned, at least the size returned by
 * sq_splitk_workspace_size(M, N, K) on the same device; owned by the caller,
 * used as scratch during the call.  Its first 256-byte-rounded block holds
 * arrival counters that must be zero before the first call (cudaMemset); a
 * call that completes leaves them zero again.  After a call that reported
 * SQ_ERR_TIMEOUT, zero the workspace before reusing it.  Calls that share a
 * workspace must not overlap on the GPU. */
sq_status sq_linear_forward_codes_splitk(const int8_t* q_pos, const int8_t* q_neg, int64_t ldq,
                                         int64_t M, int64_t K, const sq_qweight* w,
                                         const float* s_pos, const float* s_neg,
                                         const float* bias, void* y, sq_dtype yt, int64_t ldy,
                                         void* workspace, size_t workspace_bytes,
                                         sq_stream_t stream);

/* Host only: workspace bytes sq_linear_forward_codes_splitk needs for an
 * [M, K] x [N, K]^T problem on the current device (the split count depends on
 * the device's SM count).  1 <= M <= 128, N, K > 0, else SQ_ERR_INVALID_ARG. */
sq_status sq_splitk_workspace_size(int64_t M, int64_t N, int64_t K, size_t* bytes);

/* No counterpart in the SegQuant pages: an interface for callers that cannot
 * allocate device memory at call time.  The same computation and result as
 * sq_linear_forward_codes_splitk, with its workspace in a library-owned
 * file-scope device array of SQ_SPLITK_STATIC_SCRATCH_BYTES (16 MiB) per
 * device instead of a caller buffer.  The call allocates nothing (no
 * cudaMalloc, cudaFree or allocating library routine).
 * Set-up: the first call on each device, with that device current, looks up
 * the array's address (cudaGetSymbolAddress); make that first call before any
 * stream capture.  The look-up runs again on the first call after the
 * device's context has been re-created (cudaDeviceReset), since the array
 * then lives at a new address.
 * Zeroing: every call clears the array's arrival counters itself
 * (cudaMemsetAsync on `stream`) before its kernel; the partial sums need no
 * clearing.
 * Sharing: all calls on a device share the one array, so calls that overlap
 * on the GPU (on different streams without ordering between them) race; order
 * them on one stream.
 * Limit: if the split-K workspace for (M, N, K) exceeds the array even with a
 * single K split (8 * M * N bytes plus the counters), SQ_ERR_RANGE.  Other
 * requirements and errors as for sq_linear_forward_codes_splitk. */
#define SQ_SPLITK_STATIC_SCRATCH_BYTES (16u << 20)
sq_status sq_linear_forward_codes_splitk_static(const int8_t* q_pos, const int8_t* q_neg,
                                                int64_t ldq, int64_t M, int64_t K,
                                                const sq_qweight* w, const float* s_pos,
                                                const float* s_neg, const float* bias, void* y,
                                                sq_dtype yt, int64_t ldy, sq_stream_t stream);

/* Test surface: the same kernel as sq_linear_forward, but the epilogue writes
 * the raw int32 accumulators of every unit instead of Y:
 * acc[u][p][m][n], p = 0 for the (+) product, 1 for the (-) product; U units
 * (K segments for int8 weights, K/128 groups for int4 weights); int32
 * [U, 2, M, N] contiguous.  Intended for small shapes. */
sq_status sq_linear_accumulators(const void* x, sq_dtype xt, int64_t M, int64_t K, int64_t ldx,
                                 const sq_qweight* w, const float* s_pos, const float* s_neg,
                                 int32_t* acc, sq_stream_t stream);

/* Waits for `stream`, then returns and clears the device status word:
 * SQ_ERR_TIMEOUT, SQ_ERR_RANGE, SQ_ERR_CUDA (a failed synchronize), or SQ_OK.
 * The status word is per device and shared by all streams of the process. */
sq_status sq_stream_status(sq_stream_t stream);

/* Static string naming a status code. */
const char* sq_status_string(sq_status status);

/* Description of the last CUDA error that made a call of this thread return
 * SQ_ERR_CUDA ("no CUDA error" if none).  Static string; host only. */
const char* sq_last_cuda_error(void);

/* Development library only (libsegquant_dev.so, built with SQ_DEV_BUILD; the
 * product library libsegquant.so returns SQ_ERR_UNSUPPORTED and changes
 * nothing).  Test hook: the device-side wait budget in clock cycles (default
 * about one second); 0 restores the default.  Host only; affects later
 * launches of the process. */
sq_status sq_set_wait_budget(int64_t cycles);

/* Development library only (as above).  Test hook: while enabled, the GEMM
 * kernels' TMA producer issues no copy, so every consumer's bounded wait
 * expires; the launch still returns SQ_OK and sq_stream_status() then reports
 * SQ_ERR_TIMEOUT.  Host only. */
sq_status sq_debug_starve_pipeline(int32_t enable);

#ifdef __cplusplus
}
#endif

#endif /* SEGQUANT_H_ */
