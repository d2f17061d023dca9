// Host side of the C ABI declared in include/segquant.h: argument validation,
// TMA descriptor encoding and kernel launches.  One translation unit holds
// every kernel so that they share the per-device status word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>
#include <vector>

#include "segquant.h"

#include "common.cuh"
#include "gemm_dualscale.cuh"
#include "gemm_dualscale_codes.cuh"
#include "gemm_dualscale_combined.cuh"
#include "gemm_dualscale_splitk.cuh"
#include "gemm_dualscale_inplace.cuh"
#include "gemm_dualscale_pair.cuh"
#include "ptx.cuh"
#include "quant_kernels.cuh"

// Scratch of sq_linear_forward_codes_splitk_static: a file-scope device array,
// one per device (zero at module load), located with cudaGetSymbolAddress
// once per device on the first call with that device current.
static __device__ __align__(256) uint8_t g_splitk_scratch[SQ_SPLITK_STATIC_SCRATCH_BYTES];

// Activation tables of the fused producer for bf16 pre-activations: entry b of
// table a (0: SiLU, 1: GELU) is the bf16 pattern of act(z) for the bf16
// pattern b of z.  Filled once per device context by act_table_kernel.
static __device__ __align__(16) uint16_t g_act_table[2][sq::kActTableSize];

namespace {

using sq::SegBounds;

// Development build (-DSQ_DEV_BUILD, libsegquant_dev.so): the environment
// switches below select measured alternatives of the default kernels (kept so
// that tests can prove them bit-identical to the defaults) and the two test
// hooks (wait budget, starved pipeline) are live.  The product build
// (libsegquant.so) reads no environment, compiles only the default kernels
// and runs with the fixed wait budget.
#ifdef SQ_DEV_BUILD
constexpr bool kDev = true;
#else
constexpr bool kDev = false;
#endif

constexpr long long kDefaultWaitBudget = 2000000000LL;  // ~1 s of SM clock
long long g_wait_budget = kDefaultWaitBudget;            // written by the development hooks only
int g_debug_starve = 0;

// An integer development switch: the environment's value in the development
// build, `dflt` when unset and always in the product build.
int dev_switch(const char* name, int dflt) {
#ifdef SQ_DEV_BUILD
  if (const char* e = std::getenv(name)) return std::atoi(e);
#else
  (void)name;
#endif
  return dflt;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int elt_size(sq_dtype t) { return t == SQ_F32 ? 4 : 2; }
bool dtype_ok(sq_dtype t) { return t == SQ_F32 || t == SQ_BF16; }

// Segment bounds: count in [1, max_count], strictly increasing, 0 .. extent;
// interior bounds multiples of `granule` (when granule > 1).
sq_status check_segments(const sq_segments* s, int64_t extent, int max_count, int granule,
                         SegBounds* out) {
  if (s == nullptr || s->bounds == nullptr) return SQ_ERR_INVALID_ARG;
  if (s->count < 1) return SQ_ERR_INVALID_ARG;
  if (s->count > max_count) return SQ_ERR_UNSUPPORTED;
  if (s->bounds[0] != 0 || (int64_t)s->bounds[s->count] != extent) return SQ_ERR_INVALID_ARG;
  for (int i = 0; i < s->count; ++i)
    if (s->bounds[i + 1] <= s->bounds[i]) return SQ_ERR_INVALID_ARG;
  if (granule > 1)
    for (int i = 1; i < s->count; ++i)
      if (s->bounds[i] % granule != 0) return SQ_ERR_UNSUPPORTED;
  if (out != nullptr) {
    std::memset(out, 0, sizeof(*out));
    out->count = s->count;
    for (int i = 0; i <= s->count; ++i) out->b[i] = s->bounds[i];
  }
  return SQ_OK;
}

sq_status check_nseg(const sq_segments* s, int64_t N) {
  if (s == nullptr || s->bounds == nullptr || s->count < 1) return SQ_ERR_INVALID_ARG;
  if (s->bounds[0] != 0 || (int64_t)s->bounds[s->count] != N) return SQ_ERR_INVALID_ARG;
  for (int i = 0; i < s->count; ++i)
    if (s->bounds[i + 1] <= s->bounds[i]) return SQ_ERR_INVALID_ARG;
  return SQ_OK;
}

thread_local cudaError_t g_last_cuda_error = cudaSuccess;

sq_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SQ_OK;
  g_last_cuda_error = e;
  return SQ_ERR_CUDA;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2D row-major tensor, 128-byte swizzled boxes of box_inner x box_rows.
sq_status make_tmap(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                    uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner,
                    uint32_t box_rows,
                    CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto fn = encode_fn();
  if (fn == nullptr) return SQ_ERR_CUDA;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SQ_OK : SQ_ERR_CUDA;
}

// A tiled map of rank 3 or 4 over int8 data (128-byte inner boxes, 128-byte
// swizzle); strides in bytes for dimensions 1.. .
sq_status make_tmap_nd(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                       const uint64_t* strides, const uint32_t* box) {
  auto fn = encode_fn();
  if (fn == nullptr) return SQ_ERR_CUDA;
  cuuint64_t d[4], st[3];
  cuuint32_t bx[4], estr[4] = {1, 1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    if (i + 1 < rank) st[i] = strides[i];
  }
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, (cuuint32_t)rank, const_cast<void*>(base), d, st,
                  bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SQ_OK : SQ_ERR_CUDA;
}

sq_status check_qweight(const sq_qweight* w, int64_t K, SegBounds* kseg) {
  if (w == nullptr) return SQ_ERR_INVALID_ARG;
  if (w->N <= 0 || w->K <= 0 || w->K != K) return SQ_ERR_INVALID_ARG;
  if (w->codes == nullptr || w->scales == nullptr) return SQ_ERR_INVALID_ARG;
  if (!(w->bits == 8 && w->group == 0) && !(w->bits == 4 && w->group == 128))
    return SQ_ERR_UNSUPPORTED;
  if (w->N > (int64_t)INT32_MAX - 256) return SQ_ERR_RANGE;
  if (w->K > SQ_MAX_K) return SQ_ERR_RANGE;
  if (w->N % 16 != 0 || w->K % 16 != 0) return SQ_ERR_UNSUPPORTED;
  if (w->bits == 4 && w->K % 128 != 0) return SQ_ERR_UNSUPPORTED;
  sq_status s = check_segments(&w->kseg, w->K, SQ_MAX_SEGMENTS, 128, kseg);
  if (s != SQ_OK) return s;
  s = check_nseg(&w->nseg, w->N);
  if (s != SQ_OK) return s;
  if (!aligned16(w->codes) || !aligned16(w->scales)) return SQ_ERR_ALIGNMENT;
  return SQ_OK;
}

constexpr int kMaxDevices = 64;

// SM count of the current device, looked up once per device.
int num_sms() {
  static std::atomic<int> cached[kMaxDevices] = {};
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < kMaxDevices && (n = cached[dev].load(std::memory_order_relaxed)) > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  if (dev >= 0 && dev < kMaxDevices) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

// Id of the calling thread's current CUDA context, 0 when there is none (or
// it cannot be read).  Context ids are unique for the life of the process, so
// a context re-created on the same device (after cudaDeviceReset) has a new id.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (get_current(&c) != CUDA_SUCCESS || c == nullptr || get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Raises kernel KERN's dynamic shared memory limit to `bytes`, once per
// context (the attribute lasts as long as the context): later launches skip
// the call.
template <auto KERN>
cudaError_t smem_limit(int bytes) {
  static std::atomic<unsigned long long> done_ctx[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cacheable = dev >= 0 && dev < kMaxDevices;
  const unsigned long long ctx = current_context_id();
  if (cacheable && ctx != 0 && done_ctx[dev].load(std::memory_order_acquire) == ctx) return cudaSuccess;
  e = cudaFuncSetAttribute(KERN, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && cacheable && ctx != 0) done_ctx[dev].store(ctx, std::memory_order_release);
  return e;
}

template <int BN, int ASRC, typename XT, bool W4, bool ACC, bool YB, bool MULTI>
sq_status launch_gemm(const CUtensorMap& ta, const CUtensorMap& ta2, const CUtensorMap& tw,
                      sq::GemmArgs a, cudaStream_t stream) {
  using C = sq::GemmCfg<BN, ASRC, XT, W4>;
  constexpr auto kern = sq::dualscale_gemm_kernel<BN, ASRC, XT, W4, ACC, YB, MULTI>;
  cudaError_t e = smem_limit<kern>(C::SMEM_BYTES);
  if (e != cudaSuccess) return cuda_status(e);
  a.n_full = a.N / BN;
  a.tail = a.N % BN;
  a.m_tiles = (a.M + sq::BM - 1) / sq::BM;
  a.num_tiles = a.m_tiles * (a.n_full + (a.tail ? 1 : 0));
  int grid = num_sms();
  if (grid > a.num_tiles) grid = a.num_tiles;
  kern<<<grid, sq::kernel_threads(MULTI), C::SMEM_BYTES, stream>>>(ta, ta2, tw, a);
  return cuda_status(cudaGetLastError());
}

// Picks the output variant: raw accumulators (test surface) or fp32 / bf16 Y.
template <int BN, int ASRC, typename XT, bool W4, bool MULTI>
sq_status launch_out(bool acc, bool y_bf16, const CUtensorMap& ta, const CUtensorMap& ta2,
                     const CUtensorMap& tw, const sq::GemmArgs& a, cudaStream_t stream) {
  if constexpr (MULTI) {
    if (acc) return launch_gemm<BN, ASRC, XT, W4, true, false, true>(ta, ta2, tw, a, stream);
  }
  if (acc) return SQ_ERR_UNSUPPORTED;
  return y_bf16 ? launch_gemm<BN, ASRC, XT, W4, false, true, MULTI>(ta, ta2, tw, a, stream)
                : launch_gemm<BN, ASRC, XT, W4, false, false, MULTI>(ta, ta2, tw, a, stream);
}

template <int BN, bool YB, bool MULTI, int EPW>
sq_status launch_pair(const CUtensorMap& ta, const CUtensorMap& ta2, const CUtensorMap& tw,
                      const CUtensorMap& ty, sq::GemmArgs a, cudaStream_t stream) {
  using C = sq::PairCfg<BN, EPW, YB>;
  constexpr auto kern = sq::dualscale_gemm_pair_kernel<BN, YB, MULTI, EPW>;
  cudaError_t e = smem_limit<kern>(C::SMEM_BYTES);
  if (e != cudaSuccess) return cuda_status(e);
  a.n_full = a.N / BN;
  a.tail = a.N % BN;
  a.m_tiles = (a.M + sq::BM_PAIR - 1) / sq::BM_PAIR;
  a.num_tiles = a.m_tiles * (a.n_full + (a.tail ? 1 : 0));
  int pairs = num_sms() / 2;
  if (pairs > a.num_tiles) pairs = a.num_tiles;
  kern<<<2 * pairs, sq::pair_threads(EPW), C::SMEM_BYTES, stream>>>(ta, ta2, tw, ty, a);
  return cuda_status(cudaGetLastError());
}

// 2-SM pair tiles with 16 epilogue warps per CTA (32 or 64 columns per warp).
template <int BN, bool MULTI>
sq_status launch_pair_out(bool y_bf16, const CUtensorMap& ta, const CUtensorMap& ta2,
                          const CUtensorMap& tw, const CUtensorMap& ty, const sq::GemmArgs& a,
                          cudaStream_t stream) {
  return y_bf16 ? launch_pair<BN, true, MULTI, 16>(ta, ta2, tw, ty, a, stream)
                : launch_pair<BN, false, MULTI, 16>(ta, ta2, tw, ty, a, stream);
}

template <int BN, bool ACC, bool YB, bool MULTI>
sq_status launch_inplace(const CUtensorMap& tx, const CUtensorMap& tw, sq::GemmArgs a,
                         cudaStream_t stream) {
  using C = sq::InplaceCfg<BN>;
  constexpr auto kern = sq::dualscale_gemm_inplace_kernel<BN, ACC, YB, MULTI>;
  cudaError_t e = smem_limit<kern>(C::SMEM_BYTES);
  if (e != cudaSuccess) return cuda_status(e);
  a.n_full = a.N / BN;
  a.tail = a.N % BN;
  a.m_tiles = (a.M + sq::BM - 1) / sq::BM;
  a.num_tiles = a.m_tiles * (a.n_full + (a.tail ? 1 : 0));
  int grid = num_sms();
  if (grid > a.num_tiles) grid = a.num_tiles;
  kern<<<grid, sq::kernel_threads(MULTI), C::SMEM_BYTES, stream>>>(tx, tw, a);
  return cuda_status(cudaGetLastError());
}

template <int BN, bool MULTI>
sq_status launch_inplace_out(bool acc, bool y_bf16, const CUtensorMap& tx, const CUtensorMap& tw,
                             const sq::GemmArgs& a, cudaStream_t stream) {
  if constexpr (MULTI) {
    if (acc) return launch_inplace<BN, true, false, true>(tx, tw, a, stream);
  }
  if (acc) return SQ_ERR_UNSUPPORTED;
  return y_bf16 ? launch_inplace<BN, false, true, MULTI>(tx, tw, a, stream)
                : launch_inplace<BN, false, false, MULTI>(tx, tw, a, stream);
}

// Whether the GEMM from codes copies the code tiles with cp.async loader warps
// (TMA then carries only the weight tile); off unless SEGQUANT_CODES_LDA=1
// (measured slower than all-TMA loads on the DiT, MMDiT and SegLinear shapes).
bool use_codes_lda() { return dev_switch("SEGQUANT_CODES_LDA", 0) != 0; }


// k blocks per pipeline stage of the GEMM from codes (2 for TMA loads at
// BN <= 192, where two such stages fit; 1 otherwise); SEGQUANT_KPS=1 forces one.
int codes_kps() { return dev_switch("SEGQUANT_KPS", 2) == 2 ? 2 : 1; }

// Whether a single row tile of M <= 64 stacks its q+ and q- rows in one A
// tile (one MMA per k step); SEGQUANT_STACK=0 selects two 128-row code tiles.
bool use_stacked() { return dev_switch("SEGQUANT_STACK", 1) != 0; }

// Whether a small-M row tile with few N tiles splits the K range of
// each tile over a cluster of CTAs; SEGQUANT_CSPLIT=0 keeps one CTA per tile.
bool use_cluster_split() { return dev_switch("SEGQUANT_CSPLIT", 1) != 0; }

template <int BN, bool YB, bool MULTI, bool SINGLE, int EPW = sq::epi_warps(MULTI), bool LDA = false,
          int KPS = 1, int WM = 0, int STK = 0, bool CSPLIT = false>
sq_status launch_codes(const CUtensorMap& tqp, const CUtensorMap& tqn, const CUtensorMap& tw,
                       const CUtensorMap& ty, sq::GemmArgs a, cudaStream_t stream) {
  if constexpr (kDev && !LDA && KPS == 1 && WM == 0 && STK == 0 && !CSPLIT && !(MULTI && BN > 128)) {
    if (use_codes_lda()) return launch_codes<BN, YB, MULTI, SINGLE, EPW, true>(tqp, tqn, tw, ty, a, stream);
  }
  // (not for a K split: its partial sums take the room of the second k block)
  if constexpr (!LDA && KPS == 1 && WM == 0 && STK == 0 && !CSPLIT && BN <= 192 &&
                sq::codes_kps2_fits(BN, MULTI, YB, SINGLE, EPW)) {
    if (codes_kps() == 2)
      return launch_codes<BN, YB, MULTI, SINGLE, EPW, false, 2>(tqp, tqn, tw, ty, a, stream);
  }
  using C = sq::CodesCfg<BN, MULTI, YB, SINGLE, EPW, LDA, KPS, WM, STK, CSPLIT>;
  constexpr auto kern =
      sq::dualscale_gemm_codes_kernel<BN, YB, MULTI, SINGLE, EPW, LDA, KPS, WM, STK, CSPLIT>;
  cudaError_t e = smem_limit<kern>(C::SMEM_BYTES);
  if (e != cudaSuccess) return cuda_status(e);
  a.n_full = a.N / BN;
  a.tail = a.N % BN;
  a.m_tiles = (a.M + sq::BM - 1) / sq::BM;
  a.num_tiles = a.m_tiles * (a.n_full + (a.tail ? 1 : 0));
  int grid = num_sms();
  if (grid > a.num_tiles) grid = a.num_tiles;
  if constexpr (CSPLIT) grid = a.num_tiles * a.splits;   // one cluster of `splits` CTAs per tile
  // Programmatic launch: the kernel's setup (barriers, TMEM, descriptor
  // prefetch) overlaps the tail of the kernel before it in the stream; the
  // kernel waits for that kernel before touching its inputs.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)sq::codes_threads(EPW, LDA, WM == 1));
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = CSPLIT ? (unsigned)a.splits : 1u;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = CSPLIT ? 2 : 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, kern, tqp, tqn, tw, ty, a));
}

template <int BN, bool MULTI, bool SINGLE = false, int EPW = sq::epi_warps(MULTI), int WM = 0>
sq_status launch_codes_out(bool y_bf16, const CUtensorMap& tqp, const CUtensorMap& tqn,
                           const CUtensorMap& tw, const CUtensorMap& ty, const sq::GemmArgs& a,
                           cudaStream_t stream) {
  return y_bf16 ? launch_codes<BN, true, MULTI, SINGLE, EPW, false, 1, WM>(tqp, tqn, tw, ty, a, stream)
                : launch_codes<BN, false, MULTI, SINGLE, EPW, false, 1, WM>(tqp, tqn, tw, ty, a, stream);
}

// Whether int4 weights run through the GEMM from codes (unpack warps, one
// ring of stages, seeded accumulators); SEGQUANT_W4_CODES=0 selects the
// operand-ring kernel with producer warps.
bool use_codes_w4() { return dev_switch("SEGQUANT_W4_CODES", 1) != 0; }

// Whether 256-wide tiles of the GEMM from codes drain TMEM with 16 epilogue
// warps instead of 8 (one TMEM buffer at that width: the MMA waits for the
// drain); SEGQUANT_EPW16=0|1 overrides the default.
bool codes_wide_epilogue() { return dev_switch("SEGQUANT_EPW16", 1) != 0; }

// Small M (one row tile): the work is streaming the weight codes, so the tile
// width spreads N over as many SMs as possible.  Candidates 32..256 (multiples
// of 32, four epilogue warps); cost = waves x cycles per MMA, where an M = 128
// MMA takes about BN/2 cycles but no less than 48 (narrow products lose rate);
// ties go to the narrower tile (more SMs share the stream).  0 = not small.
// Whether the development switch SEGQUANT_BN_SMALL fixes the small-M tile width.
bool bn_small_forced() {
  const int v = dev_switch("SEGQUANT_BN_SMALL", 0);
  return v == 32 || v == 64 || v == 96 || v == 128;
}

int choose_bn_small(int64_t M, int64_t N) {
  if (M > sq::BM) return 0;
  {
    const int v = dev_switch("SEGQUANT_BN_SMALL", 0);
    if (v == 32 || v == 64 || v == 96 || v == 128) return v;
    if (v == -1) return 0;   // the regular tile choice
  }
  const int sms = num_sms();
  int best = 0;
  double best_cost = 0.0;
  for (int bn : {32, 64, 96, 128}) {
    const int64_t tiles = (N + bn - 1) / bn;
    const double waves = (double)((tiles + sms - 1) / sms);
    const double cost = waves * std::max(bn, 96);
    if (best == 0 || cost < best_cost) {
      best = bn;
      best_cost = cost;
    }
  }
  return best;
}

// Small M with stacked polarities (one MMA per k step for both products):
// stk = 16 for M <= 16, 64 for 16 < M <= 64 (args.a_rows = 32 or 64); two k
// blocks per stage.
template <int BN>
sq_status launch_codes_stacked(int stk, bool y_bf16, const CUtensorMap& tqp, const CUtensorMap& tqn,
                               const CUtensorMap& tw, const CUtensorMap& ty, const sq::GemmArgs& a,
                               cudaStream_t stream) {
  if (stk == 16)
    return y_bf16 ? launch_codes<BN, true, false, false, 4, false, 2, 0, 16>(tqp, tqn, tw, ty, a, stream)
                  : launch_codes<BN, false, false, false, 4, false, 2, 0, 16>(tqp, tqn, tw, ty, a, stream);
  return y_bf16 ? launch_codes<BN, true, false, false, 4, false, 2, 0, 64>(tqp, tqn, tw, ty, a, stream)
                : launch_codes<BN, false, false, false, 4, false, 2, 0, 64>(tqp, tqn, tw, ty, a, stream);
}

// Stacked rows (stk = 16: M <= 16; 64: 16 < M <= 64) with each N tile's k
// blocks shared by the a.splits CTAs of a cluster.
template <int BN>
sq_status launch_codes_split(int stk, bool y_bf16, const CUtensorMap& tqp, const CUtensorMap& tqn,
                             const CUtensorMap& tw, const CUtensorMap& ty, const sq::GemmArgs& a,
                             cudaStream_t stream) {
  if (stk == 16)
    return y_bf16
               ? launch_codes<BN, true, false, false, 4, false, 2, 0, 16, true>(tqp, tqn, tw, ty, a, stream)
               : launch_codes<BN, false, false, false, 4, false, 2, 0, 16, true>(tqp, tqn, tw, ty, a, stream);
  return y_bf16
             ? launch_codes<BN, true, false, false, 4, false, 2, 0, 64, true>(tqp, tqn, tw, ty, a, stream)
             : launch_codes<BN, false, false, false, 4, false, 2, 0, 64, true>(tqp, tqn, tw, ty, a, stream);
}

sq_status launch_codes_small_split(int bn, int stk, bool y_bf16, const CUtensorMap& tqp,
                                   const CUtensorMap& tqn, const CUtensorMap& tw,
                                   const CUtensorMap& ty, const sq::GemmArgs& a, cudaStream_t stream) {
  switch (bn) {
    case 32: return launch_codes_split<32>(stk, y_bf16, tqp, tqn, tw, ty, a, stream);
    case 64: return launch_codes_split<64>(stk, y_bf16, tqp, tqn, tw, ty, a, stream);
    case 96: return launch_codes_split<96>(stk, y_bf16, tqp, tqn, tw, ty, a, stream);
    default: return launch_codes_split<128>(stk, y_bf16, tqp, tqn, tw, ty, a, stream);
  }
}

// How many clusters of `cs` CTAs, one CTA per SM, the current device runs at
// once.  A cluster stays inside one group of SMs, so this is below
// num_sms() / cs when the groups' sizes are not multiples of cs.  0 when the
// query fails.
int max_clusters(int cs) {
  static std::atomic<int> cached[kMaxDevices][9] = {};
  int dev = 0;
  if (cs < 1 || cs > 8 || cudaGetDevice(&dev) != cudaSuccess) return 0;
  const bool cacheable = dev >= 0 && dev < kMaxDevices;
  if (cacheable) {
    const int v = cached[dev][cs].load(std::memory_order_relaxed);
    if (v != 0) return v > 0 ? v : 0;
  }
  constexpr auto kern = sq::dualscale_gemm_codes_kernel<128, true, false, false, 4, false, 2, 0, 16, true>;
  // most of an SM's shared memory: one CTA per SM whatever the tile width (the
  // attribute is an upper bound, so raising it leaves every launch valid)
  constexpr int kQuerySmem = 200 * 1024;
  int n = 0;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kQuerySmem) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cs);
    cfg.blockDim = dim3((unsigned)sq::codes_threads(4, false, false));
    cfg.dynamicSmemBytes = kQuerySmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      n = 0;
    }
  }
  if (cacheable) cached[dev][cs].store(n > 0 ? n : -1, std::memory_order_relaxed);
  return n;
}

// Small M (one row tile): the tile width and the cluster size that shares each
// N tile's k blocks.  The time of such a layer follows the number of k blocks
// a CTA streams (the stages in flight cover a fixed HBM latency each), not
// the tile width: the narrow tile `bn0` split over as many CTAs (2..8, at least
// min_kb k blocks apiece, clusters the device runs at once) as the SMs hold;
// when bn0 cannot be split and its tiles leave a fifth of the SMs idle, the
// tile of twice its width split in two or more (up to max_bn: the two-tile
// form's partial sums fit beside two stages up to 96 columns).  `forced`: keep bn0.
void choose_small_split(int64_t N, int num_kb, int bn0, bool forced, int max_bn, int min_kb, int& bn,
                        int& cs) {
  const int sms = num_sms();
  bn = bn0;
  cs = 1;
  if (bn0 > max_bn) return;
  auto split_of = [&](int b) {
    const int64_t tiles = (N + b - 1) / b;
    int c = 1;
    for (int k = 2; k <= 8; ++k)
      if (tiles * k <= sms && num_kb >= min_kb * k && tiles <= max_clusters(k)) c = k;
    return c;
  };
  cs = split_of(bn0);
  if (forced || cs > 1 || bn0 * 2 > max_bn || ((N + bn0 - 1) / bn0) * 5 >= (int64_t)sms * 4) return;
  const int c2 = split_of(bn0 * 2);
  if (c2 > 1) {
    bn = bn0 * 2;
    cs = c2;
  }
}

sq_status launch_codes_small_stacked(int bn, int stk, bool y_bf16, const CUtensorMap& tqp,
                                     const CUtensorMap& tqn, const CUtensorMap& tw,
                                     const CUtensorMap& ty, const sq::GemmArgs& a,
                                     cudaStream_t stream) {
  switch (bn) {
    case 32: return launch_codes_stacked<32>(stk, y_bf16, tqp, tqn, tw, ty, a, stream);
    case 64: return launch_codes_stacked<64>(stk, y_bf16, tqp, tqn, tw, ty, a, stream);
    case 96: return launch_codes_stacked<96>(stk, y_bf16, tqp, tqn, tw, ty, a, stream);
    default: return launch_codes_stacked<128>(stk, y_bf16, tqp, tqn, tw, ty, a, stream);
  }
}

// The two-tile form (16 < M <= 128, or M <= 64 without stacking) with each N
// tile's k blocks shared by the a.splits CTAs of a cluster.
sq_status launch_codes_small_split2(int bn, bool y_bf16, const CUtensorMap& tqp, const CUtensorMap& tqn,
                                    const CUtensorMap& tw, const CUtensorMap& ty, const sq::GemmArgs& a,
                                    cudaStream_t stream) {
#define SQ_SPLIT2(B)                                                                                  \
  return y_bf16 ? launch_codes<B, true, false, false, 4, false, 1, 0, 0, true>(tqp, tqn, tw, ty, a, stream) \
                : launch_codes<B, false, false, false, 4, false, 1, 0, 0, true>(tqp, tqn, tw, ty, a, stream)
  switch (bn) {   // (the [2][128][BN] partial sums leave room for two stages up to BN = 96)
    case 32: SQ_SPLIT2(32);
    case 64: SQ_SPLIT2(64);
    case 96: SQ_SPLIT2(96);
    default: return SQ_ERR_UNSUPPORTED;
  }
#undef SQ_SPLIT2
}

template <bool SINGLE>
sq_status launch_codes_small(int bn, bool y_bf16, const CUtensorMap& tqp, const CUtensorMap& tqn,
                             const CUtensorMap& tw, const CUtensorMap& ty, const sq::GemmArgs& a,
                             cudaStream_t stream) {
  switch (bn) {
    case 32: return launch_codes_out<32, false, SINGLE, 4>(y_bf16, tqp, tqn, tw, ty, a, stream);
    case 64: return launch_codes_out<64, false, SINGLE, 4>(y_bf16, tqp, tqn, tw, ty, a, stream);
    case 96: return launch_codes_out<96, false, SINGLE, 4>(y_bf16, tqp, tqn, tw, ty, a, stream);
    default: return launch_codes_out<128, false, SINGLE, 4>(y_bf16, tqp, tqn, tw, ty, a, stream);
  }
}

// Tensor map of Y for the TMA-store epilogue: boxes of 32 rows x 32 columns,
// bf16 rows of 64 bytes in the 64-byte swizzle, fp32 rows of 128 bytes in the
// 128-byte swizzle (the staging layout of epilogue_tma_store).
// Y for TMA stores of 32 columns x box_rows rows (32; 16 for stacked rows,
// whose warps store groups of 16 rows).
sq_status make_tmap_y(CUtensorMap* map, void* y, sq_dtype yt, int64_t M, int64_t N, int64_t ldy,
                      uint32_t box_rows = 32) {
  const bool bf = (yt == SQ_BF16);
  return make_tmap(map, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, y,
                   (uint64_t)N, (uint64_t)M, (uint64_t)(ldy * (bf ? 2 : 4)), 32, box_rows,
                   bf ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int BN, bool YB, bool MULTI>
sq_status launch_combined(const CUtensorMap& tc, const CUtensorMap& tw, sq::GemmArgs a,
                          cudaStream_t stream) {
  using C = sq::CombinedCfg<BN>;
  constexpr auto kern = sq::dualscale_gemm_combined_kernel<BN, YB, MULTI>;
  cudaError_t e = smem_limit<kern>(C::SMEM_BYTES);
  if (e != cudaSuccess) return cuda_status(e);
  a.n_full = a.N / BN;
  a.tail = a.N % BN;
  a.m_tiles = (a.M + sq::BM - 1) / sq::BM;
  a.num_tiles = a.m_tiles * (a.n_full + (a.tail ? 1 : 0));
  int grid = num_sms();
  if (grid > a.num_tiles) grid = a.num_tiles;
  kern<<<grid, sq::combined_kernel_threads(MULTI), C::SMEM_BYTES, stream>>>(tc, tw, a);
  return cuda_status(cudaGetLastError());
}

template <int BN, bool MULTI>
sq_status launch_combined_out(bool y_bf16, const CUtensorMap& tc, const CUtensorMap& tw,
                              const sq::GemmArgs& a, cudaStream_t stream) {
  return y_bf16 ? launch_combined<BN, true, MULTI>(tc, tw, a, stream)
                : launch_combined<BN, false, MULTI>(tc, tw, a, stream);
}

// Split-K plan for M <= 128: tile width, K splits and workspace layout.  Units
// (N tile, K split) are sized to fill the SMs once; every split gets at least
// one k block.
struct SplitPlan {
  int bn, splits, kb_per_split, n_tiles;
  size_t count_bytes, part_bytes;
};

SplitPlan plan_splitk(int64_t M, int64_t N, int64_t K) {
  SplitPlan p;
  p.bn = (N >= 2048) ? 256 : 128;
  p.n_tiles = (int)((N + p.bn - 1) / p.bn);
  const int num_kb = (int)((K + sq::BK - 1) / sq::BK);
  int splits = num_sms() / p.n_tiles;
  splits = std::max(1, std::min(splits, std::min(num_kb, 16)));
  p.kb_per_split = (num_kb + splits - 1) / splits;
  p.splits = (num_kb + p.kb_per_split - 1) / p.kb_per_split;
  p.count_bytes = ((size_t)p.n_tiles * 8 * sizeof(int32_t) + 255) / 256 * 256;
  p.part_bytes = (size_t)p.splits * 2 * (size_t)M * (size_t)N * sizeof(int32_t);
  return p;
}

// The split-K plan with its workspace capped at `cap` bytes: fewer K splits
// until it fits; false if even one split does not.
bool plan_splitk_capped(int64_t M, int64_t N, int64_t K, size_t cap, SplitPlan* out) {
  SplitPlan p = plan_splitk(M, N, K);
  const int num_kb = (int)((K + sq::BK - 1) / sq::BK);
  for (int want = p.splits; want >= 1; --want) {
    p.kb_per_split = (num_kb + want - 1) / want;
    p.splits = (num_kb + p.kb_per_split - 1) / p.kb_per_split;
    p.part_bytes = (size_t)p.splits * 2 * (size_t)M * (size_t)N * sizeof(int32_t);
    if (p.count_bytes + p.part_bytes <= cap) {
      *out = p;
      return true;
    }
  }
  return false;
}

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};

std::mutex g_table_mu;
const uint16_t* g_table_ptr[kMaxDevices] = {};
unsigned long long g_table_ctx[kMaxDevices] = {};

// Device address of the filled activation tables in the current context.  The
// first call per device (and per re-created context) launches the two table
// kernels on `s` and waits for them, so that calls on any stream find the
// tables complete.
sq_status act_tables(cudaStream_t s, const uint16_t** out) {
  int dev = 0;
  sq_status st = cuda_status(cudaGetDevice(&dev));
  if (st != SQ_OK) return st;
  if (dev < 0 || dev >= kMaxDevices) return SQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_table_mu);
  const unsigned long long ctx = current_context_id();
  if (g_table_ptr[dev] == nullptr || ctx == 0 || ctx != g_table_ctx[dev]) {
    void* p = nullptr;
    st = cuda_status(cudaGetSymbolAddress(&p, g_act_table));
    if (st != SQ_OK) return st;
    uint16_t* t = static_cast<uint16_t*>(p);
    sq::act_table_kernel<sq::ACT_SILU><<<sq::kActTableSize / 256, 256, 0, s>>>(t);
    sq::act_table_kernel<sq::ACT_GELU><<<sq::kActTableSize / 256, 256, 0, s>>>(t + sq::kActTableSize);
    st = cuda_status(cudaGetLastError());
    if (st != SQ_OK) return st;
    st = cuda_status(cudaStreamSynchronize(s));
    if (st != SQ_OK) return st;
    g_table_ptr[dev] = t;
    g_table_ctx[dev] = current_context_id();
  }
  *out = g_table_ptr[dev];
  return SQ_OK;
}

// Device address of g_splitk_scratch in the current device's context: looked
// up with cudaGetSymbolAddress on the first call per device and again whenever
// the device's context has changed since (the array lives in the context's
// copy of the module).
sq_status static_scratch(void** out) {
  int dev = 0;
  sq_status st = cuda_status(cudaGetDevice(&dev));
  if (st != SQ_OK) return st;
  if (dev < 0 || dev >= kMaxDevices) return SQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  const unsigned long long ctx = current_context_id();
  if (g_scratch_ptr[dev] == nullptr || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    st = cuda_status(cudaGetSymbolAddress(&p, g_splitk_scratch));
    if (st != SQ_OK) return st;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = current_context_id();   // the lookup made the context current
  }
  *out = g_scratch_ptr[dev];
  return SQ_OK;
}

template <int BN, bool YB>
sq_status launch_splitk(const CUtensorMap& tqp, const CUtensorMap& tqn, const CUtensorMap& tw,
                        sq::GemmArgs a, cudaStream_t stream) {
  using C = sq::SplitKCfg<BN>;
  constexpr auto kern = sq::dualscale_gemm_splitk_kernel<BN, YB>;
  cudaError_t e = smem_limit<kern>(C::SMEM_BYTES);
  if (e != cudaSuccess) return cuda_status(e);
  int grid = num_sms();
  const int units = a.num_tiles * a.splits;
  if (grid > units) grid = units;
  kern<<<grid, sq::codes_kernel_threads(false), C::SMEM_BYTES, stream>>>(tqp, tqn, tw, a);
  return cuda_status(cudaGetLastError());
}

// Whether the GEMM from int8 codes runs the one-ring kernel (codes and weight
// tile in one stage); SEGQUANT_CODES_RING=0 selects the kernel with separate
// operand rings.
bool use_codes_ring() { return dev_switch("SEGQUANT_CODES_RING", 1) != 0; }

// Whether the fused path quantizes bf16 activations in place (one ring of
// stages): int8 weights; SEGQUANT_INPLACE=0 selects the separate-ring kernel.
bool use_inplace(bool w4) {
  if (w4) return false;
  return dev_switch("SEGQUANT_INPLACE", 1) != 0;
}

// Whether the GEMM from codes runs on CTA pairs (2-SM UMMA): int8 weights and a
// last tile width that is a multiple of 32 (pair MMA N granularity).
// SEGQUANT_PAIR=0|1 overrides the default.
bool use_pair(int64_t N, bool w4) {
  if (!kDev || w4 || N % 32 != 0) return false;
  return dev_switch("SEGQUANT_PAIR", 0) != 0;
}

// Output-tile width.  Several units per tile need double-buffered TMEM, which
// caps BN at 128; fp32 activation stages leave room for BN = 128 only.
// Otherwise BN in {128, 192, 256} minimises a makespan model of the snake
// schedule: the busiest CTA's tile columns divided by the measured per-column
// efficiency of that width.  Two calibrations, each measured on B200:
//  * the GEMM from codes (one stage ring, two k blocks per stage, 16 epilogue
//    warps at BN = 256): 0.70, 0.79, 0.90, and the last, narrower tile column
//    costs its own width (full tiles are scheduled first);
//  * the other kernels: 0.55, 0.70, 0.81, and the last tile costs a full one.
// SEGQUANT_BN=128|192|256 overrides the choice (a tuning knob).
int choose_bn(int64_t M, int64_t N, bool multi, bool f32x, bool codes_ring) {
  if (multi || f32x) return 128;
  {
    const int v = dev_switch("SEGQUANT_BN", 0);
    if (v == 128 || v == 192 || v == 256) return v;
  }
  const int sms = num_sms();
  const int64_t m_tiles = (M + sq::BM - 1) / sq::BM;
  std::vector<double> load(sms);
  auto cost = [&](int64_t bn, double eff) {
    std::fill(load.begin(), load.end(), 0.0);
    const int64_t n_full = N / bn, tail = N % bn;
    const int64_t full_tiles = m_tiles * n_full;
    const int64_t tiles = full_tiles + (tail ? m_tiles : 0);
    for (int64_t idx = 0; idx < tiles; ++idx) {
      const int64_t it = idx / sms, pos = idx % sms;
      const int64_t cta = (it & 1) ? sms - 1 - pos : pos;
      load[cta] += (double)(idx < full_tiles || !codes_ring ? bn : tail) / eff;
    }
    return *std::max_element(load.begin(), load.end());
  };
  const double c128 = cost(128, codes_ring ? 0.70 : 0.55);
  const double c192 = cost(192, codes_ring ? 0.79 : 0.70);
  const double c256 = cost(256, codes_ring ? 0.90 : 0.81);
  if (c256 <= c192 && c256 <= c128) return 256;
  return c192 <= c128 ? 192 : 128;
}

// Tile width of the GEMM from codes when a tile folds several units (K
// segments, int8 weights): 128 (two TMEM buffers, 16 epilogue warps), 192
// (one buffer, 12 warps of 64 columns) or 256 (one buffer, 16 warps of 64
// columns).  Per k block a tile needs 32 KiB of codes plus BN x 128 bytes of
// weights per 4 x BN tensor-core cycles, against about 51 bytes per clock that
// an SM's TMA engine delivers, so wider tiles run closer to the MMA rate
// (about 0.53, 0.70 and 0.80 of it) but leave more tiles unbalanced over the
// SMs; the makespan of the snake schedule over those rates decides.
// SEGQUANT_BN overrides.
int choose_bn_multi(int64_t M, int64_t N) {
  {
    const int v = dev_switch("SEGQUANT_BN", 0);
    if (v == 128 || v == 192 || v == 256) return v;
  }
  const int sms = num_sms();
  const int64_t m_tiles = (M + sq::BM - 1) / sq::BM;
  std::vector<double> load(sms);
  auto cost = [&](int64_t bn, double eff) {
    std::fill(load.begin(), load.end(), 0.0);
    const int64_t n_full = N / bn, tail = N % bn;
    const int64_t full_tiles = m_tiles * n_full;
    const int64_t tiles = full_tiles + (tail ? m_tiles : 0);
    for (int64_t idx = 0; idx < tiles; ++idx) {
      const int64_t it = idx / sms, pos = idx % sms;
      const int64_t cta = (it & 1) ? sms - 1 - pos : pos;
      load[cta] += (double)(idx < full_tiles ? bn : std::max<int64_t>(tail, bn / 2)) / eff;
    }
    return *std::max_element(load.begin(), load.end());
  };
  const double c128 = cost(128, 0.53), c192 = cost(192, 0.70), c256 = cost(256, 0.80);
  if (c256 <= c192 && c256 <= c128) return 256;
  return c192 <= c128 ? 192 : 128;
}

// Codes of X: q+ and q- (CODES_DUAL), the combined code c = q+ + q-
// (CODES_COMBINED) or the single-scale code (CODES_SINGLE), the last two
// written to q_pos.
sq_status quantize_codes(const void* x, sq_dtype xt, int64_t M, int64_t K, int64_t ldx,
                         const sq_segments* kseg, const float* s_pos, const float* s_neg,
                         int8_t* q_pos, int8_t* q_neg, int64_t ldq, int mode, cudaStream_t s) {
  const bool combined = (mode == sq::CODES_COMBINED || mode == sq::CODES_SINGLE ||
                         mode == sq::CODES_SILU || mode == sq::CODES_GELU);
  if (!dtype_ok(xt) || M < 0 || K <= 0 || ldx < K || ldq < K) return SQ_ERR_INVALID_ARG;
  if (K > SQ_MAX_K) return SQ_ERR_RANGE;
  SegBounds sb;
  sq_status st = check_segments(kseg, K, SQ_MAX_SEGMENTS, 128, &sb);
  if (st != SQ_OK) return st;
  if (K % 16 != 0) return SQ_ERR_UNSUPPORTED;
  if (M > (int64_t)INT32_MAX) return SQ_ERR_RANGE;
  if (M == 0) return SQ_OK;
  if (x == nullptr || s_pos == nullptr || s_neg == nullptr || q_pos == nullptr ||
      (!combined && q_neg == nullptr))
    return SQ_ERR_INVALID_ARG;
  const int xe = elt_size(xt);
  if (!aligned16(x) || (ldx * xe) % 16 != 0 || !aligned16(q_pos) ||
      (!combined && !aligned16(q_neg)) || ldq % 16 != 0)
    return SQ_ERR_ALIGNMENT;
  const int64_t groups = K / 16;
  const int gx = (int)((groups + 31) / 32);
  int64_t gy = (M + 7) / 8;
  // sixteen 256-thread blocks per SM: two full waves of eight resident blocks
  // (a grid just past that would leave a few blocks for a third)
  const int64_t cap = (int64_t)num_sms() * 16 / gx;
  if (gy > cap) gy = cap;
  if (gy > 65535) gy = 65535;
  if (gy < 1) gy = 1;
  dim3 grid(gx, (unsigned)gy), block(32, 8);
  using bf = __nv_bfloat16;
  if (mode == sq::CODES_COMBINED) {
    if (xt == SQ_BF16)
      sq::quantize_activations_combined_kernel<bf, sq::CODES_COMBINED><<<grid, block, 0, s>>>(
          static_cast<const bf*>(x), (int32_t)M, (int32_t)K, ldx, sb, s_pos, s_neg, q_pos, ldq);
    else
      sq::quantize_activations_combined_kernel<float, sq::CODES_COMBINED><<<grid, block, 0, s>>>(
          static_cast<const float*>(x), (int32_t)M, (int32_t)K, ldx, sb, s_pos, s_neg, q_pos, ldq);
  } else if ((mode == sq::CODES_SILU || mode == sq::CODES_GELU) && xt == SQ_BF16) {
    // bf16 pre-activations: through the activation table in shared memory
    const uint16_t* tables = nullptr;
    st = act_tables(s, &tables);
    if (st != SQ_OK) return st;
    const uint16_t* lut = tables + (mode == sq::CODES_GELU ? sq::kActTableSize : 0);
    constexpr int kTableSmem = sq::kActTableSize * 2;
    constexpr auto kern = sq::quantize_combined_act_table_kernel;
    st = cuda_status(smem_limit<kern>(kTableSmem));
    if (st != SQ_OK) return st;
    // One 1024-thread block per SM (the table fills its shared memory): at most
    // one block per SM, so no SM runs a second one after the others finish.
    const int64_t ty = std::min<int64_t>((M + 31) / 32,
                                         std::max<int64_t>(1, num_sms() / gx));
    dim3 tgrid(gx, (unsigned)std::min<int64_t>(ty, 65535)), tblock(32, 32);
    kern<<<tgrid, tblock, kTableSmem, s>>>(static_cast<const bf*>(x), (int32_t)M, (int32_t)K, ldx,
                                           sb, s_pos, s_neg, lut, q_pos, ldq);
  } else if (mode == sq::CODES_SILU) {
    if (xt == SQ_BF16)
      sq::quantize_activations_combined_kernel<bf, sq::CODES_SILU><<<grid, block, 0, s>>>(
          static_cast<const bf*>(x), (int32_t)M, (int32_t)K, ldx, sb, s_pos, s_neg, q_pos, ldq);
    else
      sq::quantize_activations_combined_kernel<float, sq::CODES_SILU><<<grid, block, 0, s>>>(
          static_cast<const float*>(x), (int32_t)M, (int32_t)K, ldx, sb, s_pos, s_neg, q_pos, ldq);
  } else if (mode == sq::CODES_GELU) {
    if (xt == SQ_BF16)
      sq::quantize_activations_combined_kernel<bf, sq::CODES_GELU><<<grid, block, 0, s>>>(
          static_cast<const bf*>(x), (int32_t)M, (int32_t)K, ldx, sb, s_pos, s_neg, q_pos, ldq);
    else
      sq::quantize_activations_combined_kernel<float, sq::CODES_GELU><<<grid, block, 0, s>>>(
          static_cast<const float*>(x), (int32_t)M, (int32_t)K, ldx, sb, s_pos, s_neg, q_pos, ldq);
  } else if (mode == sq::CODES_SINGLE) {
    if (xt == SQ_BF16)
      sq::quantize_activations_combined_kernel<bf, sq::CODES_SINGLE><<<grid, block, 0, s>>>(
          static_cast<const bf*>(x), (int32_t)M, (int32_t)K, ldx, sb, s_pos, s_neg, q_pos, ldq);
    else
      sq::quantize_activations_combined_kernel<float, sq::CODES_SINGLE><<<grid, block, 0, s>>>(
          static_cast<const float*>(x), (int32_t)M, (int32_t)K, ldx, sb, s_pos, s_neg, q_pos, ldq);
  } else if (mode == sq::CODES_HADAMARD) {
    if (xt == SQ_BF16)
      sq::quantize_activations_hadamard_kernel<bf><<<grid, block, 0, s>>>(
          static_cast<const bf*>(x), (int32_t)M, (int32_t)K, ldx, sb, s_pos, s_neg, q_pos, q_neg,
          ldq);
    else
      sq::quantize_activations_hadamard_kernel<float><<<grid, block, 0, s>>>(
          static_cast<const float*>(x), (int32_t)M, (int32_t)K, ldx, sb, s_pos, s_neg, q_pos, q_neg,
          ldq);
  } else {
    if (xt == SQ_BF16)
      sq::quantize_activations_kernel<bf><<<grid, block, 0, s>>>(
          static_cast<const bf*>(x), (int32_t)M, (int32_t)K, ldx, sb, s_pos, s_neg, q_pos, q_neg,
          ldq);
    else
      sq::quantize_activations_kernel<float><<<grid, block, 0, s>>>(
          static_cast<const float*>(x), (int32_t)M, (int32_t)K, ldx, sb, s_pos, s_neg, q_pos, q_neg,
          ldq);
  }
  return cuda_status(cudaGetLastError());
}

// Hadamard: q+/q- codes of the block-Hadamard-transformed activations, against
// the rotated int4 weight codes (int8 [N][ldr]) with the int4 group scales.
enum class ASource { X, Codes, Combined, Single, Hadamard };

sq_status gemm_common(ASource src, const void* x, sq_dtype xt, const int8_t* q_pos,
                      const int8_t* q_neg, int64_t ldq, int64_t M, int64_t K, int64_t ldx,
                      const sq_qweight* w, const float* s_pos, const float* s_neg,
                      const float* bias, void* y, sq_dtype yt, int64_t ldy, int32_t* acc,
                      cudaStream_t stream, const int8_t* w_rot = nullptr, int64_t ldr = 0) {
  const bool had = (src == ASource::Hadamard);
  const bool dual_codes = (src == ASource::Codes) || had;   // q+ and q- tensors
  if (src == ASource::X && !dtype_ok(xt)) return SQ_ERR_INVALID_ARG;
  if (acc == nullptr && !dtype_ok(yt)) return SQ_ERR_INVALID_ARG;
  if (M < 0 || K <= 0) return SQ_ERR_INVALID_ARG;
  SegBounds kseg;
  sq_status st = check_qweight(w, K, &kseg);
  if (st != SQ_OK) return st;
  const int64_t N = w->N;
  if (src == ASource::X && ldx < K) return SQ_ERR_INVALID_ARG;
  if (src != ASource::X && ldq < K) return SQ_ERR_INVALID_ARG;
  if ((src == ASource::Combined || src == ASource::Single) && w->bits != 8) return SQ_ERR_UNSUPPORTED;
  if (had && (w->bits != 4 || acc != nullptr)) return SQ_ERR_UNSUPPORTED;
  if (had && (w_rot == nullptr || ldr < K)) return SQ_ERR_INVALID_ARG;
  if (had && (!aligned16(w_rot) || ldr % 16 != 0)) return SQ_ERR_ALIGNMENT;
  if (acc == nullptr && ldy < N) return SQ_ERR_INVALID_ARG;
  if (M > (int64_t)INT32_MAX - 2 * sq::BM) return SQ_ERR_RANGE;
  if (M == 0) return SQ_OK;
  if (s_pos == nullptr || s_neg == nullptr) return SQ_ERR_INVALID_ARG;
  if (src == ASource::X && x == nullptr) return SQ_ERR_INVALID_ARG;
  if (dual_codes && (q_pos == nullptr || q_neg == nullptr)) return SQ_ERR_INVALID_ARG;
  if ((src == ASource::Combined || src == ASource::Single) && q_pos == nullptr) return SQ_ERR_INVALID_ARG;
  if (acc == nullptr && y == nullptr) return SQ_ERR_INVALID_ARG;
  if (src == ASource::X && (!aligned16(x) || (ldx * elt_size(xt)) % 16 != 0)) return SQ_ERR_ALIGNMENT;
  if (dual_codes && (!aligned16(q_pos) || !aligned16(q_neg) || ldq % 16 != 0))
    return SQ_ERR_ALIGNMENT;
  if ((src == ASource::Combined || src == ASource::Single) && (!aligned16(q_pos) || ldq % 16 != 0))
    return SQ_ERR_ALIGNMENT;
  if (acc == nullptr && (!aligned16(y) || (ldy * elt_size(yt)) % 16 != 0)) return SQ_ERR_ALIGNMENT;
  if (acc != nullptr && !aligned16(acc)) return SQ_ERR_ALIGNMENT;
  if (bias != nullptr && !aligned16(bias)) return SQ_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(s_pos) & 3u) || (reinterpret_cast<uintptr_t>(s_neg) & 3u))
    return SQ_ERR_ALIGNMENT;

  const bool w4 = (w->bits == 4);
  const bool multi = w4 || kseg.count > 1;
  const bool f32x = (src == ASource::X && xt == SQ_F32);
  const bool pair = (src == ASource::Codes) && use_pair(N, w4);
  const bool codes_ring = (src == ASource::Codes) && !w4 && !pair && acc == nullptr && use_codes_ring();
  int BN = (acc != nullptr || multi) ? 128 : choose_bn(M, N, multi, f32x, codes_ring);
  if (multi && codes_ring) BN = choose_bn_multi(M, N);   // several K segments, from codes
  // one row tile, one unit per tile, GEMM from codes: narrow tiles over all SMs
  int bn_small = (!multi && acc == nullptr && (src == ASource::Codes || src == ASource::Single) &&
                        !(src == ASource::Codes && use_pair(N, w4)) && use_codes_ring())
                           ? choose_bn_small(M, N) : 0;
  if (bn_small) BN = bn_small;
  if (pair && acc == nullptr) BN = dev_switch("SEGQUANT_BN", 256) == 128 ? 128 : 256;
  // One row tile of fewer than BM rows, read by the GEMM from codes: code boxes
  // of M rows rounded up to 16 instead of mostly out-of-bounds 128-row boxes.
  const bool codes_w4 = (src == ASource::Codes) && w4 && !pair && acc == nullptr && use_codes_w4();
  const bool codes_kernel = (src == ASource::Single) || codes_ring || codes_w4 || had;
  // M <= 64 rows of q+ and q- stacked in one A tile (P = 16, 32 or 64 rows each)
  const bool stacked = bn_small && src == ASource::Codes && M <= 64 && use_stacked();
  // each N tile's k blocks shared by a cluster of split_cs CTAs, on a tile
  // width chosen for it
  int split_cs = 1;
  if (bn_small && src == ASource::Codes && !pair && use_cluster_split()) {
    int sbn = bn_small;
    // (k blocks per CTA: at least 2 with 16 stacked rows, 5 otherwise -- below
    // that the exchange of partial sums costs more than the split saves)
    choose_small_split(N, (int)((K + sq::BK - 1) / sq::BK), bn_small, bn_small_forced(),
                       stacked ? 128 : 96, (stacked && M <= 16) ? 2 : 5, sbn, split_cs);
    if (split_cs > 1) {
      bn_small = sbn;
      BN = sbn;
    }
  }
  const int a_rows = stacked ? (int)((M + 15) / 16 * 16)   // groups of 16 rows
                     : (codes_kernel && M < sq::BM) ? (int)((M + 15) / 16 * 16) : sq::BM;
  CUtensorMap ta, ta2, tw;
  if (src == ASource::X) {
    const int xe = elt_size(xt);
    st = make_tmap(&ta, xt == SQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                   x, (uint64_t)K, (uint64_t)M, (uint64_t)(ldx * xe), 128 / xe, sq::BM);
    if (st != SQ_OK) return st;
    ta2 = ta;
  } else {
    // (stacked rows: boxes of 16 rows, one per group and polarity)
    const uint32_t box_rows = stacked ? 16u : (uint32_t)a_rows;
    st = make_tmap(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_pos, (uint64_t)K, (uint64_t)M,
                   (uint64_t)ldq, 128, box_rows);
    if (st != SQ_OK) return st;
    if (dual_codes) {
      st = make_tmap(&ta2, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_neg, (uint64_t)K, (uint64_t)M,
                     (uint64_t)ldq, 128, box_rows);
      if (st != SQ_OK) return st;
    } else {
      ta2 = ta;
    }
  }
  if (had)   // rotated codes, int8 rows of ldr bytes
    st = make_tmap(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_rot, (uint64_t)K, (uint64_t)N,
                   (uint64_t)ldr, 128, (uint32_t)BN);
  else if (w4)
    st = make_tmap(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes, (uint64_t)(K / 2), (uint64_t)N,
                   (uint64_t)(K / 2), 64, (uint32_t)BN, CU_TENSOR_MAP_SWIZZLE_NONE);
  else
    st = make_tmap(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes, (uint64_t)K, (uint64_t)N,
                   (uint64_t)K, 128, (uint32_t)(pair ? BN / 2 : BN));
  if (st != SQ_OK) return st;

  sq::GemmArgs a;
  std::memset(&a, 0, sizeof(a));
  a.M = (int32_t)M;
  a.N = (int32_t)N;
  a.K = (int32_t)K;
  a.num_kb = (int32_t)((K + sq::BK - 1) / sq::BK);
  a.bits = w->bits;
  a.kseg = kseg;
  a.s_pos = s_pos;
  a.s_neg = s_neg;
  a.wscales = w->scales;
  a.bias = bias;
  a.y = y;
  a.ldy = ldy;
  a.acc_out = acc;
  a.wait_budget = kDev ? g_wait_budget : kDefaultWaitBudget;
  a.starve = kDev ? g_debug_starve : 0;
  a.a_pos = q_pos;
  a.a_neg = q_neg;
  a.lda = ldq;
  a.a_rows = a_rows;
  // stacked rows: the whole groups of 16 rows of both polarities in one box
  // of a 4-D map (no row past the whole groups is addressed), and a partial
  // last group in two boxes of a 3-D map over all M rows (rows past M read as
  // zeros).  Both maps start at the lower of the two code tensors (planes q+,
  // q- or q-, q+), whose distance must be a multiple of 16 bytes.
  if (stacked) {
    const uintptr_t pp = reinterpret_cast<uintptr_t>(q_pos), pn = reinterpret_cast<uintptr_t>(q_neg);
    const bool neg_first = pn < pp;
    const uintptr_t gap = neg_first ? pp - pn : pn - pp;
    const void* low = neg_first ? static_cast<const void*>(q_neg) : static_cast<const void*>(q_pos);
    if (gap > 0 && gap % 16 == 0 && gap < (1ull << 40)) {
      const int64_t whole = M / 16;
      if (whole > 0) {
        const uint64_t cd[4] = {(uint64_t)K, 16, 2, (uint64_t)whole};
        const uint64_t cs[3] = {(uint64_t)ldq, (uint64_t)gap, (uint64_t)(16 * ldq)};
        const uint32_t cb[4] = {(uint32_t)sq::BK, 16, 2, (uint32_t)whole};
        st = make_tmap_nd(&ta, low, 4, cd, cs, cb);
        if (st != SQ_OK) return st;
      }
      if (M % 16 != 0) {
        const uint64_t cd[3] = {(uint64_t)K, (uint64_t)M, 2};
        const uint64_t cs[2] = {(uint64_t)ldq, (uint64_t)gap};
        const uint32_t cb[3] = {(uint32_t)sq::BK, 16, 1};
        st = make_tmap_nd(&ta2, low, 3, cd, cs, cb);
        if (st != SQ_OK) return st;
      }
      a.code_box4 = (M % 16 != 0) ? 2 : 1;
      a.code_neg_first = neg_first ? 1 : 0;
    }
  }

  using bf = __nv_bfloat16;
  constexpr int AX = sq::ASRC_X, AC = sq::ASRC_CODES;
  const bool yb = (yt == SQ_BF16);
  const bool ac = (acc != nullptr);
  if (had) {
    CUtensorMap ty;
    st = make_tmap_y(&ty, y, yt, M, N, ldy);
    if (st != SQ_OK) return st;
    return launch_codes_out<128, true, false, sq::epi_warps(true), 2>(yb, ta, ta2, tw, ty, a, stream);
  }
  if (src == ASource::Single) {
    CUtensorMap ty;
    st = make_tmap_y(&ty, y, yt, M, N, ldy);
    if (st != SQ_OK) return st;
    if (multi) return launch_codes_out<128, true, true>(yb, ta, ta, tw, ty, a, stream);
    if (bn_small) return launch_codes_small<true>(bn_small, yb, ta, ta, tw, ty, a, stream);
    if (BN == 256) return launch_codes_out<256, false, true>(yb, ta, ta, tw, ty, a, stream);
    if (BN == 192) return launch_codes_out<192, false, true>(yb, ta, ta, tw, ty, a, stream);
    return launch_codes_out<128, false, true>(yb, ta, ta, tw, ty, a, stream);
  }
  if (src == ASource::Combined) {
    if (multi) return launch_combined_out<128, true>(yb, ta, tw, a, stream);
    if (BN == 256) return launch_combined_out<256, false>(yb, ta, tw, a, stream);
    if (BN == 192) return launch_combined_out<192, false>(yb, ta, tw, a, stream);
    return launch_combined_out<128, false>(yb, ta, tw, a, stream);
  }
  if constexpr (kDev) {   // 2-SM pair tiles: a measured alternative
    if (pair) {
      CUtensorMap ty;
      st = make_tmap_y(&ty, y, yt, M, N, ldy);
      if (st != SQ_OK) return st;
      if (multi) {
        if (BN == 256) return launch_pair_out<256, true>(yb, ta, ta2, tw, ty, a, stream);
        return launch_pair_out<128, true>(yb, ta, ta2, tw, ty, a, stream);
      }
      if (BN == 256) return launch_pair_out<256, false>(yb, ta, ta2, tw, ty, a, stream);
      return launch_pair_out<128, false>(yb, ta, ta2, tw, ty, a, stream);
    }
  }
  if (src == ASource::Codes) {
    if (codes_w4) {
      CUtensorMap ty;
      st = make_tmap_y(&ty, y, yt, M, N, ldy);
      if (st != SQ_OK) return st;
      return launch_codes_out<128, true, false, sq::epi_warps(true), 1>(yb, ta, ta2, tw, ty, a, stream);
    }
    if constexpr (kDev) {   // int4 through the operand-ring kernel
      if (w4) return launch_out<128, AC, bf, true, true>(ac, yb, ta, ta2, tw, a, stream);
    }
    if (!ac && use_codes_ring()) {
      CUtensorMap ty;
      st = make_tmap_y(&ty, y, yt, M, N, ldy);
      if (st != SQ_OK) return st;
      if (multi) {
        if (BN == 256) return launch_codes_out<256, true, false, 16>(yb, ta, ta2, tw, ty, a, stream);
        if (BN == 192) return launch_codes_out<192, true, false, 12>(yb, ta, ta2, tw, ty, a, stream);
        return launch_codes_out<128, true>(yb, ta, ta2, tw, ty, a, stream);
      }
      if (stacked) {
        CUtensorMap ty16;   // the warps store groups of 16 rows
        st = make_tmap_y(&ty16, y, yt, M, N, ldy, 16);
        if (st != SQ_OK) return st;
        if (split_cs > 1) {   // CTA r of a cluster: k blocks [r*kb/cs, (r+1)*kb/cs)
          a.splits = split_cs;
          return launch_codes_small_split(bn_small, a_rows <= 16 ? 16 : 64, yb, ta, ta2, tw, ty16, a,
                                          stream);
        }
        return launch_codes_small_stacked(bn_small, a_rows <= 16 ? 16 : 64, yb, ta, ta2, tw, ty16, a,
                                          stream);
      }
      if (bn_small && split_cs > 1) {   // two-tile form, k blocks shared by a cluster
        a.splits = split_cs;
        return launch_codes_small_split2(bn_small, yb, ta, ta2, tw, ty, a, stream);
      }
      if (bn_small) return launch_codes_small<false>(bn_small, yb, ta, ta2, tw, ty, a, stream);
      if (BN == 256 && codes_wide_epilogue())
        return launch_codes_out<256, false, false, 16>(yb, ta, ta2, tw, ty, a, stream);
      if constexpr (kDev) {   // eight epilogue warps at BN = 256
        if (BN == 256) return launch_codes_out<256, false>(yb, ta, ta2, tw, ty, a, stream);
      }
      if (BN == 192) return launch_codes_out<192, false>(yb, ta, ta2, tw, ty, a, stream);
      return launch_codes_out<128, false>(yb, ta, ta2, tw, ty, a, stream);
    }
    if constexpr (kDev) {   // separate operand rings
      if (multi || ac) return launch_out<128, AC, bf, false, true>(ac, yb, ta, ta2, tw, a, stream);
      if (BN == 256) return launch_out<256, AC, bf, false, false>(ac, yb, ta, ta2, tw, a, stream);
      if (BN == 192) return launch_out<192, AC, bf, false, false>(ac, yb, ta, ta2, tw, a, stream);
      return launch_out<128, AC, bf, false, false>(ac, yb, ta, ta2, tw, a, stream);
    }
    return SQ_ERR_UNSUPPORTED;   // not reached in the product build
  }
  if (f32x) {
    if (w4) return launch_out<128, AX, float, true, true>(ac, yb, ta, ta2, tw, a, stream);
    if (multi || ac) return launch_out<128, AX, float, false, true>(ac, yb, ta, ta2, tw, a, stream);
    return launch_out<128, AX, float, false, false>(ac, yb, ta, ta2, tw, a, stream);
  }
  if (w4) return launch_out<128, AX, bf, true, true>(ac, yb, ta, ta2, tw, a, stream);
  if (use_inplace(w4)) {
    if (multi || ac) return launch_inplace_out<128, true>(ac, yb, ta, tw, a, stream);
    if (BN == 256) return launch_inplace_out<256, false>(ac, yb, ta, tw, a, stream);
    if (BN == 192) return launch_inplace_out<192, false>(ac, yb, ta, tw, a, stream);
    return launch_inplace_out<128, false>(ac, yb, ta, tw, a, stream);
  }
  if constexpr (kDev) {   // bf16 activations quantized by producer warps into separate tiles
    if (multi || ac) return launch_out<128, AX, bf, false, true>(ac, yb, ta, ta2, tw, a, stream);
    if (BN == 256) return launch_out<256, AX, bf, false, false>(ac, yb, ta, ta2, tw, a, stream);
    if (BN == 192) return launch_out<192, AX, bf, false, false>(ac, yb, ta, ta2, tw, a, stream);
    return launch_out<128, AX, bf, false, false>(ac, yb, ta, ta2, tw, a, stream);
  }
  return SQ_ERR_UNSUPPORTED;   // not reached in the product build
}

}  // namespace

extern "C" {

const char* sq_last_cuda_error(void) {
  return g_last_cuda_error == cudaSuccess ? "no CUDA error" : cudaGetErrorString(g_last_cuda_error);
}

const char* sq_status_string(sq_status s) {
  switch (s) {
    case SQ_OK: return "SQ_OK";
    case SQ_ERR_INVALID_ARG: return "SQ_ERR_INVALID_ARG";
    case SQ_ERR_ALIGNMENT: return "SQ_ERR_ALIGNMENT";
    case SQ_ERR_UNSUPPORTED: return "SQ_ERR_UNSUPPORTED";
    case SQ_ERR_RANGE: return "SQ_ERR_RANGE";
    case SQ_ERR_CUDA: return "SQ_ERR_CUDA";
    case SQ_ERR_TIMEOUT: return "SQ_ERR_TIMEOUT";
  }
  return "SQ_UNKNOWN_STATUS";
}

sq_status sq_set_wait_budget(int64_t cycles) {
  if constexpr (!kDev) return SQ_ERR_UNSUPPORTED;
  g_wait_budget = cycles > 0 ? cycles : kDefaultWaitBudget;
  return SQ_OK;
}

sq_status sq_debug_starve_pipeline(int32_t enable) {
  if constexpr (!kDev) return SQ_ERR_UNSUPPORTED;
  g_debug_starve = enable != 0;
  return SQ_OK;
}

sq_status sq_qweight_sizes(int32_t bits, int64_t N, int64_t K, int32_t J, int32_t group,
                           size_t* code_bytes, size_t* scale_bytes) {
  if (code_bytes == nullptr || scale_bytes == nullptr) return SQ_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0 || J < 1) return SQ_ERR_INVALID_ARG;
  if (bits == 8 && group == 0) {
    if (J > SQ_MAX_SEGMENTS) return SQ_ERR_UNSUPPORTED;
    *code_bytes = (size_t)N * (size_t)K;
    *scale_bytes = (size_t)J * (size_t)N * sizeof(float);
    return SQ_OK;
  }
  if (bits == 4 && group == 128) {
    if (K % 128 != 0) return SQ_ERR_UNSUPPORTED;
    *code_bytes = (size_t)N * (size_t)(K / 2);
    *scale_bytes = (size_t)N * (size_t)(K / 128) * 2;
    return SQ_OK;
  }
  return SQ_ERR_UNSUPPORTED;
}

sq_status sq_calibrate(const void* x, sq_dtype xt, int64_t rows, int64_t K, int64_t ldx,
                       const sq_segments* kseg, float* s_pos, float* s_neg, sq_stream_t stream) {
  if (!dtype_ok(xt) || rows < 0 || K <= 0 || ldx < K) return SQ_ERR_INVALID_ARG;
  if (s_pos == nullptr || s_neg == nullptr) return SQ_ERR_INVALID_ARG;
  if (K > SQ_MAX_K) return SQ_ERR_RANGE;
  SegBounds sb;
  sq_status st = check_segments(kseg, K, SQ_MAX_SEGMENTS, 128, &sb);
  if (st != SQ_OK) return st;
  const int xe = elt_size(xt);
  if (K % (16 / xe) != 0) return SQ_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(s_pos) & 3u) || (reinterpret_cast<uintptr_t>(s_neg) & 3u))
    return SQ_ERR_ALIGNMENT;
  if (rows > 0) {
    if (x == nullptr) return SQ_ERR_INVALID_ARG;
    if (!aligned16(x) || (ldx * xe) % 16 != 0) return SQ_ERR_ALIGNMENT;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t bytes = sizeof(float) * (size_t)sb.count;
  sq_status ms = cuda_status(cudaMemsetAsync(s_pos, 0, bytes, s));
  if (ms != SQ_OK) return ms;
  ms = cuda_status(cudaMemsetAsync(s_neg, 0, bytes, s));
  if (ms != SQ_OK) return ms;
  if (rows == 0) return SQ_OK;
  const int64_t nvec = K / (16 / xe);
  const int gx = (int)((nvec + 31) / 32);
  int64_t gy = (rows + 7) / 8;
  // eight resident 256-thread blocks per SM; every block streams an equal
  // share of the rows, so the grid fills the SMs once and no block runs in a
  // second wave after the others
  int64_t cap = (int64_t)num_sms() * 8 / gx;
  if (cap < 1) cap = 1;
  if (gy > cap) gy = cap;
  if (gy > 65535) gy = 65535;
  dim3 grid(gx, (unsigned)gy), block(32, 8);
  if (xt == SQ_BF16)
    sq::calibrate_kernel<__nv_bfloat16><<<grid, block, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), rows, K, ldx, sb, s_pos, s_neg);
  else
    sq::calibrate_kernel<float><<<grid, block, 0, s>>>(static_cast<const float*>(x), rows, K, ldx,
                                                       sb, s_pos, s_neg);
  return cuda_status(cudaGetLastError());
}

sq_status sq_quantize_weights(const void* w, sq_dtype wt, int64_t N, int64_t K, int64_t ldw,
                              const sq_qweight* out, sq_stream_t stream) {
  if (!dtype_ok(wt) || w == nullptr || out == nullptr) return SQ_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0 || ldw < K) return SQ_ERR_INVALID_ARG;
  if (out->N != N) return SQ_ERR_INVALID_ARG;
  SegBounds kseg;
  sq_status st = check_qweight(out, K, &kseg);
  if (st != SQ_OK) return st;
  if (!aligned16(w) || (ldw * elt_size(wt)) % 16 != 0) return SQ_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (out->bits == 8) {
    const int64_t blocks = N * kseg.count;
    if (blocks > INT32_MAX) return SQ_ERR_RANGE;
    if (wt == SQ_BF16)
      sq::quantize_weights_w8_kernel<__nv_bfloat16><<<(unsigned)blocks, 128, 0, s>>>(
          static_cast<const __nv_bfloat16*>(w), N, K, ldw, kseg, static_cast<int8_t*>(out->codes),
          static_cast<float*>(out->scales));
    else
      sq::quantize_weights_w8_kernel<float><<<(unsigned)blocks, 128, 0, s>>>(
          static_cast<const float*>(w), N, K, ldw, kseg, static_cast<int8_t*>(out->codes),
          static_cast<float*>(out->scales));
  } else {
    const int64_t warps = N * (K / 128);
    const int blocks = (int)((warps * 32 + 255) / 256);
    if (wt == SQ_BF16)
      sq::quantize_weights_w4_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(w), N, K, ldw, static_cast<uint8_t*>(out->codes),
          static_cast<__half*>(out->scales));
    else
      sq::quantize_weights_w4_kernel<float><<<blocks, 256, 0, s>>>(
          static_cast<const float*>(w), N, K, ldw, static_cast<uint8_t*>(out->codes),
          static_cast<__half*>(out->scales));
  }
  return cuda_status(cudaGetLastError());
}

sq_status sq_quantize_activations(const void* x, sq_dtype xt, int64_t M, int64_t K, int64_t ldx,
                                  const sq_segments* kseg, const float* s_pos,
                                  const float* s_neg, int8_t* q_pos, int8_t* q_neg, int64_t ldq,
                                  sq_stream_t stream) {
  return quantize_codes(x, xt, M, K, ldx, kseg, s_pos, s_neg, q_pos, q_neg, ldq, sq::CODES_DUAL,
                        reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_quantize_activations_combined(const void* x, sq_dtype xt, int64_t M, int64_t K,
                                           int64_t ldx, const sq_segments* kseg,
                                           const float* s_pos, const float* s_neg, int8_t* c,
                                           int64_t ldc, sq_stream_t stream) {
  return quantize_codes(x, xt, M, K, ldx, kseg, s_pos, s_neg, c, nullptr, ldc,
                        sq::CODES_COMBINED, reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_quantize_activations_single(const void* x, sq_dtype xt, int64_t M, int64_t K,
                                         int64_t ldx, const sq_segments* kseg, const float* s_pos,
                                         const float* s_neg, int8_t* c, int64_t ldc,
                                         sq_stream_t stream) {
  return quantize_codes(x, xt, M, K, ldx, kseg, s_pos, s_neg, c, nullptr, ldc, sq::CODES_SINGLE,
                        reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_linear_forward(const void* x, sq_dtype xt, int64_t M, int64_t K, int64_t ldx,
                            const sq_qweight* w, const float* s_pos, const float* s_neg,
                            const float* bias, void* y, sq_dtype yt, int64_t ldy,
                            sq_stream_t stream) {
  return gemm_common(ASource::X, x, xt, nullptr, nullptr, 0, M, K, ldx, w, s_pos, s_neg, bias, y,
                     yt, ldy, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_linear_forward_codes(const int8_t* q_pos, const int8_t* q_neg, int64_t ldq,
                                  int64_t M, int64_t K, const sq_qweight* w, const float* s_pos,
                                  const float* s_neg, const float* bias, void* y, sq_dtype yt,
                                  int64_t ldy, sq_stream_t stream) {
  return gemm_common(ASource::Codes, nullptr, SQ_BF16, q_pos, q_neg, ldq, M, K, 0, w, s_pos,
                     s_neg, bias, y, yt, ldy, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_linear_forward_combined(const int8_t* c, int64_t ldc, int64_t M, int64_t K,
                                     const sq_qweight* w, const float* s_pos, const float* s_neg,
                                     const float* bias, void* y, sq_dtype yt, int64_t ldy,
                                     sq_stream_t stream) {
  return gemm_common(ASource::Combined, nullptr, SQ_BF16, c, nullptr, ldc, M, K, 0, w, s_pos,
                     s_neg, bias, y, yt, ldy, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_linear_forward_single(const int8_t* c, int64_t ldc, int64_t M, int64_t K,
                                   const sq_qweight* w, const float* s_pos, const float* s_neg,
                                   const float* bias, void* y, sq_dtype yt, int64_t ldy,
                                   sq_stream_t stream) {
  return gemm_common(ASource::Single, nullptr, SQ_BF16, c, nullptr, ldc, M, K, 0, w, s_pos, s_neg,
                     bias, y, yt, ldy, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// Calibration of transformed rows (XH, or the activation of a pre-activation):
// xf is sq::CODES_HADAMARD, sq::CODES_SILU or sq::CODES_GELU.
sq_status calibrate_transformed(const void* x, sq_dtype xt, int64_t rows, int64_t K, int64_t ldx,
                                const sq_segments* kseg, float* s_pos, float* s_neg, int xf,
                                cudaStream_t s) {
  if (!dtype_ok(xt) || rows < 0 || K <= 0 || ldx < K) return SQ_ERR_INVALID_ARG;
  if (s_pos == nullptr || s_neg == nullptr) return SQ_ERR_INVALID_ARG;
  if (K > SQ_MAX_K) return SQ_ERR_RANGE;
  SegBounds sb;
  sq_status st = check_segments(kseg, K, SQ_MAX_SEGMENTS, 128, &sb);
  if (st != SQ_OK) return st;
  if (K % 16 != 0) return SQ_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(s_pos) & 3u) || (reinterpret_cast<uintptr_t>(s_neg) & 3u))
    return SQ_ERR_ALIGNMENT;
  const int xe = elt_size(xt);
  if (rows > 0) {
    if (x == nullptr) return SQ_ERR_INVALID_ARG;
    if (!aligned16(x) || (ldx * xe) % 16 != 0) return SQ_ERR_ALIGNMENT;
  }
  const size_t bytes = sizeof(float) * (size_t)sb.count;
  sq_status ms = cuda_status(cudaMemsetAsync(s_pos, 0, bytes, s));
  if (ms != SQ_OK) return ms;
  ms = cuda_status(cudaMemsetAsync(s_neg, 0, bytes, s));
  if (ms != SQ_OK) return ms;
  if (rows == 0) return SQ_OK;
  const int64_t groups = K / 16;
  const int gx = (int)((groups + 31) / 32);
  int64_t gy = (rows + 7) / 8;
  const int64_t cap = std::max<int64_t>(1, (int64_t)num_sms() * 8 / gx);   // one wave
  if (gy > cap) gy = cap;
  if (gy > 65535) gy = 65535;
  if (gy < 1) gy = 1;
  dim3 grid(gx, (unsigned)gy), block(32, 8);
  using bf = __nv_bfloat16;
  const bf* xb = static_cast<const bf*>(x);
  const float* xf32 = static_cast<const float*>(x);
  const int32_t k32 = (int32_t)K;
  if (xf == sq::CODES_SILU) {
    if (xt == SQ_BF16)
      sq::calibrate_transformed_kernel<bf, sq::CODES_SILU><<<grid, block, 0, s>>>(xb, rows, k32, ldx, sb, s_pos, s_neg);
    else
      sq::calibrate_transformed_kernel<float, sq::CODES_SILU><<<grid, block, 0, s>>>(xf32, rows, k32, ldx, sb, s_pos, s_neg);
  } else if (xf == sq::CODES_GELU) {
    if (xt == SQ_BF16)
      sq::calibrate_transformed_kernel<bf, sq::CODES_GELU><<<grid, block, 0, s>>>(xb, rows, k32, ldx, sb, s_pos, s_neg);
    else
      sq::calibrate_transformed_kernel<float, sq::CODES_GELU><<<grid, block, 0, s>>>(xf32, rows, k32, ldx, sb, s_pos, s_neg);
  } else {
    if (xt == SQ_BF16)
      sq::calibrate_transformed_kernel<bf><<<grid, block, 0, s>>>(xb, rows, k32, ldx, sb, s_pos, s_neg);
    else
      sq::calibrate_transformed_kernel<float><<<grid, block, 0, s>>>(xf32, rows, k32, ldx, sb, s_pos, s_neg);
  }
  return cuda_status(cudaGetLastError());
}

int act_mode(sq_act act) {
  return act == SQ_ACT_SILU ? sq::CODES_SILU : (act == SQ_ACT_GELU ? sq::CODES_GELU : -1);
}

}  // namespace

extern "C" {

sq_status sq_calibrate_hadamard(const void* x, sq_dtype xt, int64_t rows, int64_t K, int64_t ldx,
                                const sq_segments* kseg, float* s_pos, float* s_neg,
                                sq_stream_t stream) {
  return calibrate_transformed(x, xt, rows, K, ldx, kseg, s_pos, s_neg, sq::CODES_HADAMARD,
                               reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_calibrate_act(const void* z, sq_dtype zt, sq_act act, int64_t rows, int64_t K,
                           int64_t ldz, const sq_segments* kseg, float* s_pos, float* s_neg,
                           sq_stream_t stream) {
  const int mode = act_mode(act);
  if (mode < 0) return SQ_ERR_INVALID_ARG;
  return calibrate_transformed(z, zt, rows, K, ldz, kseg, s_pos, s_neg, mode,
                               reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_quantize_activations_combined_act(const void* z, sq_dtype zt, sq_act act, int64_t M,
                                               int64_t K, int64_t ldz, const sq_segments* kseg,
                                               const float* s_pos, const float* s_neg, int8_t* c,
                                               int64_t ldc, sq_stream_t stream) {
  const int mode = act_mode(act);
  if (mode < 0) return SQ_ERR_INVALID_ARG;
  return quantize_codes(z, zt, M, K, ldz, kseg, s_pos, s_neg, c, nullptr, ldc, mode,
                        reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_quantize_activations_hadamard(const void* x, sq_dtype xt, int64_t M, int64_t K,
                                           int64_t ldx, const sq_segments* kseg,
                                           const float* s_pos, const float* s_neg, int8_t* q_pos,
                                           int8_t* q_neg, int64_t ldq, sq_stream_t stream) {
  return quantize_codes(x, xt, M, K, ldx, kseg, s_pos, s_neg, q_pos, q_neg, ldq,
                        sq::CODES_HADAMARD, reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_rotate_weights_hadamard(const sq_qweight* w, int8_t* w_rot, int64_t ldr,
                                     sq_stream_t stream) {
  if (w == nullptr || w_rot == nullptr) return SQ_ERR_INVALID_ARG;
  SegBounds kseg;
  sq_status st = check_qweight(w, w->K, &kseg);
  if (st != SQ_OK) return st;
  if (w->bits != 4) return SQ_ERR_UNSUPPORTED;
  if (ldr < w->K) return SQ_ERR_INVALID_ARG;
  if (!aligned16(w_rot) || ldr % 16 != 0) return SQ_ERR_ALIGNMENT;
  const int64_t tasks = w->N * (w->K / 16);
  const int64_t blocks = (tasks + 255) / 256;
  if (blocks > INT32_MAX) return SQ_ERR_RANGE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  sq::rotate_weights_hadamard_kernel<<<(unsigned)blocks, 256, 0, s>>>(
      static_cast<const uint8_t*>(w->codes), w->N, w->K, w_rot, ldr);
  return cuda_status(cudaGetLastError());
}

sq_status sq_linear_forward_codes_hadamard(const int8_t* q_pos, const int8_t* q_neg, int64_t ldq,
                                           int64_t M, int64_t K, const sq_qweight* w,
                                           const int8_t* w_rot, int64_t ldr, const float* s_pos,
                                           const float* s_neg, const float* bias, void* y,
                                           sq_dtype yt, int64_t ldy, sq_stream_t stream) {
  return gemm_common(ASource::Hadamard, nullptr, SQ_BF16, q_pos, q_neg, ldq, M, K, 0, w, s_pos,
                     s_neg, bias, y, yt, ldy, nullptr, reinterpret_cast<cudaStream_t>(stream),
                     w_rot, ldr);
}

sq_status sq_splitk_workspace_size(int64_t M, int64_t N, int64_t K, size_t* bytes) {
  if (bytes == nullptr || M < 1 || M > 128 || N <= 0 || K <= 0) return SQ_ERR_INVALID_ARG;
  const SplitPlan p = plan_splitk(M, N, K);
  *bytes = p.count_bytes + p.part_bytes;
  return SQ_OK;
}

sq_status sq_linear_forward_codes_splitk(const int8_t* q_pos, const int8_t* q_neg, int64_t ldq,
                                         int64_t M, int64_t K, const sq_qweight* w,
                                         const float* s_pos, const float* s_neg,
                                         const float* bias, void* y, sq_dtype yt, int64_t ldy,
                                         void* workspace, size_t workspace_bytes,
                                         sq_stream_t stream) {
  if (!dtype_ok(yt) || M < 0 || K <= 0 || ldq < K) return SQ_ERR_INVALID_ARG;
  SegBounds kseg;
  sq_status st = check_qweight(w, K, &kseg);
  if (st != SQ_OK) return st;
  const int64_t N = w->N;
  if (w->bits != 8 || kseg.count != 1 || M > 128) return SQ_ERR_UNSUPPORTED;
  if (ldy < N) return SQ_ERR_INVALID_ARG;
  if (M == 0) return SQ_OK;
  if (q_pos == nullptr || q_neg == nullptr || s_pos == nullptr || s_neg == nullptr ||
      y == nullptr || workspace == nullptr)
    return SQ_ERR_INVALID_ARG;
  if (!aligned16(q_pos) || !aligned16(q_neg) || ldq % 16 != 0 || !aligned16(y) ||
      (ldy * elt_size(yt)) % 16 != 0 || (bias != nullptr && !aligned16(bias)) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      (reinterpret_cast<uintptr_t>(s_pos) & 3u) || (reinterpret_cast<uintptr_t>(s_neg) & 3u))
    return SQ_ERR_ALIGNMENT;
  const SplitPlan p = plan_splitk(M, N, K);
  if (workspace_bytes < p.count_bytes + p.part_bytes) return SQ_ERR_INVALID_ARG;
  CUtensorMap ta, ta2, tw;
  st = make_tmap(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_pos, (uint64_t)K, (uint64_t)M,
                 (uint64_t)ldq, 128, sq::BM);
  if (st != SQ_OK) return st;
  st = make_tmap(&ta2, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_neg, (uint64_t)K, (uint64_t)M,
                 (uint64_t)ldq, 128, sq::BM);
  if (st != SQ_OK) return st;
  st = make_tmap(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes, (uint64_t)K, (uint64_t)N,
                 (uint64_t)K, 128, (uint32_t)p.bn);
  if (st != SQ_OK) return st;
  sq::GemmArgs a;
  std::memset(&a, 0, sizeof(a));
  a.M = (int32_t)M;
  a.N = (int32_t)N;
  a.K = (int32_t)K;
  a.num_kb = (int32_t)((K + sq::BK - 1) / sq::BK);
  a.bits = 8;
  a.kseg = kseg;
  a.m_tiles = 1;
  a.n_full = (int32_t)(N / p.bn);
  a.tail = (int32_t)(N % p.bn);
  a.num_tiles = p.n_tiles;
  a.s_pos = s_pos;
  a.s_neg = s_neg;
  a.wscales = w->scales;
  a.bias = bias;
  a.y = y;
  a.ldy = ldy;
  a.wait_budget = kDev ? g_wait_budget : kDefaultWaitBudget;
  a.starve = kDev ? g_debug_starve : 0;
  a.splits = p.splits;
  a.kb_per_split = p.kb_per_split;
  a.ws_count = static_cast<int32_t*>(workspace);
  a.ws_part = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) + p.count_bytes);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool yb = (yt == SQ_BF16);
  if (p.bn == 256) return yb ? launch_splitk<256, true>(ta, ta2, tw, a, s) : launch_splitk<256, false>(ta, ta2, tw, a, s);
  return yb ? launch_splitk<128, true>(ta, ta2, tw, a, s) : launch_splitk<128, false>(ta, ta2, tw, a, s);
}

sq_status sq_linear_forward_codes_splitk_static(const int8_t* q_pos, const int8_t* q_neg,
                                                int64_t ldq, int64_t M, int64_t K,
                                                const sq_qweight* w, const float* s_pos,
                                                const float* s_neg, const float* bias, void* y,
                                                sq_dtype yt, int64_t ldy, sq_stream_t stream) {
  if (!dtype_ok(yt) || M < 0 || K <= 0 || ldq < K) return SQ_ERR_INVALID_ARG;
  SegBounds kseg;
  sq_status st = check_qweight(w, K, &kseg);
  if (st != SQ_OK) return st;
  const int64_t N = w->N;
  if (w->bits != 8 || kseg.count != 1 || M > 128) return SQ_ERR_UNSUPPORTED;
  if (ldy < N) return SQ_ERR_INVALID_ARG;
  if (M == 0) return SQ_OK;
  if (q_pos == nullptr || q_neg == nullptr || s_pos == nullptr || s_neg == nullptr || y == nullptr)
    return SQ_ERR_INVALID_ARG;
  if (!aligned16(q_pos) || !aligned16(q_neg) || ldq % 16 != 0 || !aligned16(y) ||
      (ldy * elt_size(yt)) % 16 != 0 || (bias != nullptr && !aligned16(bias)) ||
      (reinterpret_cast<uintptr_t>(s_pos) & 3u) || (reinterpret_cast<uintptr_t>(s_neg) & 3u))
    return SQ_ERR_ALIGNMENT;
  SplitPlan p;
  if (!plan_splitk_capped(M, N, K, SQ_SPLITK_STATIC_SCRATCH_BYTES, &p)) return SQ_ERR_RANGE;
  void* scratch = nullptr;
  st = static_scratch(&scratch);
  if (st != SQ_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the arrival counters start every call at zero
  st = cuda_status(cudaMemsetAsync(scratch, 0, p.count_bytes, s));
  if (st != SQ_OK) return st;
  CUtensorMap ta, ta2, tw;
  st = make_tmap(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_pos, (uint64_t)K, (uint64_t)M,
                 (uint64_t)ldq, 128, sq::BM);
  if (st != SQ_OK) return st;
  st = make_tmap(&ta2, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_neg, (uint64_t)K, (uint64_t)M,
                 (uint64_t)ldq, 128, sq::BM);
  if (st != SQ_OK) return st;
  st = make_tmap(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes, (uint64_t)K, (uint64_t)N,
                 (uint64_t)K, 128, (uint32_t)p.bn);
  if (st != SQ_OK) return st;
  sq::GemmArgs a;
  std::memset(&a, 0, sizeof(a));
  a.M = (int32_t)M;
  a.N = (int32_t)N;
  a.K = (int32_t)K;
  a.num_kb = (int32_t)((K + sq::BK - 1) / sq::BK);
  a.bits = 8;
  a.kseg = kseg;
  a.m_tiles = 1;
  a.n_full = (int32_t)(N / p.bn);
  a.tail = (int32_t)(N % p.bn);
  a.num_tiles = p.n_tiles;
  a.s_pos = s_pos;
  a.s_neg = s_neg;
  a.wscales = w->scales;
  a.bias = bias;
  a.y = y;
  a.ldy = ldy;
  a.wait_budget = kDev ? g_wait_budget : kDefaultWaitBudget;
  a.starve = kDev ? g_debug_starve : 0;
  a.splits = p.splits;
  a.kb_per_split = p.kb_per_split;
  a.ws_count = static_cast<int32_t*>(scratch);
  a.ws_part = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(scratch) + p.count_bytes);
  const bool yb = (yt == SQ_BF16);
  if (p.bn == 256) return yb ? launch_splitk<256, true>(ta, ta2, tw, a, s) : launch_splitk<256, false>(ta, ta2, tw, a, s);
  return yb ? launch_splitk<128, true>(ta, ta2, tw, a, s) : launch_splitk<128, false>(ta, ta2, tw, a, s);
}

sq_status sq_linear_accumulators(const void* x, sq_dtype xt, int64_t M, int64_t K, int64_t ldx,
                                 const sq_qweight* w, const float* s_pos, const float* s_neg,
                                 int32_t* acc, sq_stream_t stream) {
  if (acc == nullptr) return SQ_ERR_INVALID_ARG;
  return gemm_common(ASource::X, x, xt, nullptr, nullptr, 0, M, K, ldx, w, s_pos, s_neg, nullptr,
                     nullptr, SQ_F32, 0, acc, reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_stream_status(sq_stream_t stream) {
  if (cuda_status(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream))) != SQ_OK)
    return SQ_ERR_CUDA;
  unsigned int v = 0;
  if (cuda_status(cudaMemcpyFromSymbol(&v, sq::g_status, sizeof(v))) != SQ_OK) return SQ_ERR_CUDA;
  if (v != 0) {
    const unsigned int zero = 0;
    if (cuda_status(cudaMemcpyToSymbol(sq::g_status, &zero, sizeof(zero))) != SQ_OK) return SQ_ERR_CUDA;
  }
  if (v & sq::SQ_STATUS_TIMEOUT) return SQ_ERR_TIMEOUT;
  if (v & sq::SQ_STATUS_RANGE) return SQ_ERR_RANGE;
  return SQ_OK;
}

}  // extern "C"
