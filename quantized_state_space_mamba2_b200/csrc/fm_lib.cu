// fm_lib.cu -- libfastmamba.so: the C ABI (include/fastmamba.h), host-side
// validation, TMA descriptors, the mixer composition and the calibration.
//
// Every step of the hot path runs in the kernels included below; this file
// only checks arguments, carves the caller's workspace and launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <memory>
#include <mutex>
#include <string>
#include <type_traits>
#include <vector>

#include "../../include/fastmamba.h"

#include "fm_common.cuh"
#include "k_conv.cuh"
#include "k_gemm.cuh"
#include "k_rows.cuh"
#include "k_scan.cuh"
#include "k_scan2.cuh"
#include "k_ssd.cuh"
#include "k_lq.cuh"

using namespace fm;

// ------------------------------------------------------------------ errors
static thread_local char tl_msg[512] = "";

static fm_status fail(fm_status s, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
static fm_status fail(fm_status s, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(tl_msg, sizeof(tl_msg), fmt, ap);
  va_end(ap);
  return s;
}

#define FM_CHECK_CUDA(expr)                                                          \
  do {                                                                               \
    cudaError_t e_ = (expr);                                                         \
    if (e_ != cudaSuccess)                                                           \
      return fail(FM_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(e_));             \
  } while (0)

#define FM_TRY(expr)                   \
  do {                                 \
    fm_status s_ = (expr);             \
    if (s_ != FM_OK) return s_;        \
  } while (0)

static fm_status launched(const char *what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FM_ERR_CUDA, "launch of %s: %s", what, cudaGetErrorString(e));
  return FM_OK;
}

// Programmatic dependent launch of the hot-path kernels, process-wide (off by
// default): with it a kernel may be scheduled while its predecessor in the
// stream drains; every kernel launched this way waits (pdl_wait) before its
// first global memory access.
static std::atomic<int> g_pdl{1};

extern "C" fm_status fm_set_pdl(int enable) {
  if (enable != 0 && enable != 1) return fail(FM_ERR_INVALID_ARG, "fm_set_pdl: enable must be 0 or 1");
  g_pdl.store(enable, std::memory_order_relaxed);
  return FM_OK;
}

// Set when this thread has just made a stream wait for an event of another
// stream (a pipelined stack's hand-over): the next launch then carries no
// programmatic-serialisation attribute, so that under stream capture no
// programmatic edge can reach the other stream's kernel and every kernel
// that reads a handed-over state waits for its writer's completion.
static thread_local bool t_after_cross_wait = false;

template <typename... KArgs, typename... Args>
static fm_status launch_ex(const char *name, void (*kern)(KArgs...), dim3 grid, dim3 block,
                           size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};  // no attributes unless set below
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  // never for the sequential scan, whose CTAs launched early land unevenly
  // on SMs still busy with the prep kernel (measured 232 -> 355 us per 130M
  // layer), nor for the gate after it, whose early CTAs would share the
  // issue-bound scan's SMs while they wait
  const bool placed = std::strcmp(name, "k_scan_seq") == 0 ||
                      std::strcmp(name, "k_gate_norm_quant") == 0;
  const bool after_wait = t_after_cross_wait;
  t_after_cross_wait = false;
  cfg.numAttrs = g_pdl.load(std::memory_order_relaxed) && !placed && !after_wait ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e != cudaSuccess) return fail(FM_ERR_CUDA, "launch of %s: %s", name, cudaGetErrorString(e));
  return FM_OK;
}

extern "C" const char *fm_status_string(fm_status s) {
  switch (s) {
    case FM_OK: return "FM_OK";
    case FM_ERR_INVALID_ARG: return "FM_ERR_INVALID_ARG";
    case FM_ERR_SHAPE: return "FM_ERR_SHAPE";
    case FM_ERR_ALIGNMENT: return "FM_ERR_ALIGNMENT";
    case FM_ERR_WORKSPACE: return "FM_ERR_WORKSPACE";
    case FM_ERR_NONFINITE: return "FM_ERR_NONFINITE";
    case FM_ERR_TIMEOUT: return "FM_ERR_TIMEOUT";
    case FM_ERR_CUDA: return "FM_ERR_CUDA";
    case FM_ERR_UNSUPPORTED: return "FM_ERR_UNSUPPORTED";
  }
  return "FM_ERR_UNKNOWN";
}

extern "C" const char *fm_last_error(void) { return tl_msg; }
extern "C" int fm_version(void) { return 100; }

extern "C" fm_status fm_set_fault_injection(int stall_mask, uint64_t wait_limit_ns) {
  if (stall_mask & ~(kStallGemm | kStallScan))
    return fail(FM_ERR_INVALID_ARG, "fm_set_fault_injection: unknown stall bits 0x%x", stall_mask);
  const unsigned long long lim = wait_limit_ns ? (unsigned long long)wait_limit_ns : kWaitLimitNs;
  if (lim > kWaitLimitNs)
    return fail(FM_ERR_INVALID_ARG, "fm_set_fault_injection: limit above the default %llu ns",
                kWaitLimitNs);
  FM_CHECK_CUDA(cudaMemcpyToSymbol(g_test_stall, &stall_mask, sizeof(stall_mask)));
  FM_CHECK_CUDA(cudaMemcpyToSymbol(g_wait_limit_ns, &lim, sizeof(lim)));
  return FM_OK;
}

extern "C" fm_status fm_sync_status(fm_stream stream) {
  FM_CHECK_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
  unsigned int word = 0, zero = 0;
  FM_CHECK_CUDA(cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)));
  if (word) {
    FM_CHECK_CUDA(cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)));
    if (word & kErrTimeout) return fail(FM_ERR_TIMEOUT, "a bounded device wait gave up");
    if (word & kErrNonfinite)
      return fail(FM_ERR_NONFINITE, "a non-finite value (NaN or Inf) reached an int8 quantiser");
  }
  return FM_OK;
}

// ------------------------------------------------------------------ checks
static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define NEED(p)                                                                   \
  do {                                                                            \
    if (!(p)) return fail(FM_ERR_INVALID_ARG, "%s: %s is null", __func__, #p);    \
    if (!aligned16(p))                                                            \
      return fail(FM_ERR_ALIGNMENT, "%s: %s is not 16-byte aligned", __func__, #p); \
  } while (0)
#define OPT(p)                                                                    \
  do {                                                                            \
    if ((p) && !aligned16(p))                                                     \
      return fail(FM_ERR_ALIGNMENT, "%s: %s is not 16-byte aligned", __func__, #p); \
  } while (0)

struct Dims {
  int dm = 0, di = 0, hd = 0, ds = 0, nh = 0, cc = 0, n_in = 0;  // filled by check_shape
};

static fm_status check_shape(const fm_shape *s, Dims *d, const char *fn) {
  if (!s) return fail(FM_ERR_INVALID_ARG, "%s: shape is null", fn);
  if (s->headdim != 64 || s->d_state != 128 || s->ngroups != 1 || s->d_conv != 4)
    return fail(FM_ERR_SHAPE, "%s: need headdim 64, d_state 128, ngroups 1, d_conv 4", fn);
  if (s->d_model <= 0 || s->d_model % 256 || s->d_model > 256 * kMaxBlocks || s->d_inner <= 0 ||
      s->d_inner % 256 || s->d_inner > 256 * kMaxBlocks)
    return fail(FM_ERR_SHAPE, "%s: d_model and d_inner must be positive multiples of 256, <= %d",
                fn, 256 * kMaxBlocks);
  d->dm = s->d_model;
  d->di = s->d_inner;
  d->hd = s->headdim;
  d->ds = s->d_state;
  d->nh = s->d_inner / s->headdim;
  d->cc = s->d_inner + 2 * s->d_state;
  d->n_in = 2 * s->d_inner + 2 * s->d_state + d->nh;
  return FM_OK;
}

extern "C" fm_exp_layout fm_exp_table_layout(const fm_shape *shape) {
  fm_exp_layout L;
  std::memset(&L, 0, sizeof(L));
  if (!shape || shape->headdim <= 0) return L;
  const int nh = shape->d_inner / shape->headdim;
  const int cc = shape->d_inner + 2 * shape->d_state;
  L.e_u = 0;
  L.e_w = cc;
  L.e_o = 2 * cc;
  L.e_x = 3 * cc;
  L.e_B = 3 * cc + nh;
  L.e_C = 3 * cc + nh + 1;
  L.e_h = 3 * cc + nh + 2;
  L.e_y = 3 * cc + 2 * nh + 2;
  L.e_D = 3 * cc + 3 * nh + 2;
  L.e_g = 3 * cc + 4 * nh + 2;
  L.size = 3 * cc + 4 * nh + 3;
  return L;
}

// ------------------------------------------------------------------ TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// int8 K-major [rows, K] -> tiles of box_rows x 128 bytes, 128-byte swizzle;
// rows beyond the tensor read as zero.
static fm_status make_tmap(CUtensorMap *tm, const int8_t *ptr, long long rows, long long K,
                           int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(FM_ERR_UNSUPPORTED, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K};
  cuuint32_t box[2] = {(cuuint32_t)kGemmBK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FM_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return FM_OK;
}

// 2-D output map for the GEMM epilogue's TMA stores: rows of `cols` elements
// `row_bytes` apart, boxes of 32 x 32 elements.  fp32 boxes are 128 bytes wide
// and use the 128B swizzle (matching the epilogue's staging layout); int8 boxes
// are 32 bytes wide, unswizzled.
static fm_status make_tmap_out(CUtensorMap *tm, void *ptr, bool f32, long long cols, long long rows,
                               long long row_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(FM_ERR_UNSUPPORTED, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(tm, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, ptr,
                  dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FM_ERR_CUDA, "cuTensorMapEncodeTiled (output) failed (%d)", (int)r);
  return FM_OK;
}

static bool aligned16p(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Output maps for the persistent kernel's TMA-store epilogue; ep.tma_store
// stays 0 (per-thread stores) where a map cannot describe the output (raw
// accumulators requested, or a row stride that is not a multiple of 16 bytes).
static fm_status gemm_output_maps(GemmEpilogue &ep, CUtensorMap (&tm)[3], const CUtensorMap &dummy) {
  ep.tma_store = 0;
  for (auto &t : tm) t = dummy;
  if (ep.acc_out) return FM_OK;
  if (ep.mode == 0) {
    if ((ep.N * 4) % 16 || !aligned16p(ep.Y)) return FM_OK;
    FM_TRY(make_tmap_out(&tm[0], ep.Y, true, ep.N, ep.M, ep.N * 4));
  } else {
    if ((ep.di * 4) % 16 || ep.cc % 16 || (ep.nh * 4) % 16 || ep.di % 32 || ep.cc % 32 ||
        !aligned16p(ep.z) || !aligned16p(ep.xbc) || !aligned16p(ep.dt))
      return FM_OK;
    FM_TRY(make_tmap_out(&tm[0], ep.z, true, ep.di, ep.M, (long long)ep.di * 4));
    FM_TRY(make_tmap_out(&tm[1], ep.xbc, false, ep.cc, ep.M, ep.cc));
    FM_TRY(make_tmap_out(&tm[2], ep.dt, true, ep.nh, ep.M, (long long)ep.nh * 4));
  }
  ep.tma_store = 1;
  return FM_OK;
}

// ------------------------------------------------------------------ launches
static int sm_count();

// Split-K for the small-grid kernel: enough K slices that the grid reaches
// about two CTAs per SM, every slice at least one 128-deep block.  Returns the
// number of slices (1: no split) and the blocks per slice.
static int gemm_splits(long long M, long long N, long long K, int BN, int sms, int *kbs) {
  const long long base = ((M + kGemmBM - 1) / kGemmBM) * ((N + BN - 1) / BN);
  const int nkb = (int)(K / kGemmBK);
  long long S = (2LL * sms + base - 1) / base;
  if (S > nkb) S = nkb;
  if (S < 1) S = 1;
  *kbs = (int)((nkb + S - 1) / S);
  return (nkb + *kbs - 1) / *kbs;
}
// Split-K of the small-grid GEMMs, process-wide: off by default (measured
// slower than the unsplit kernel at the 130M out_proj and the 2.7B decode
// GEMMs: the per-element atomics and the separate dequantising pass cost more
// than the extra CTAs gain).
static std::atomic<int> g_gemm_splitk{0};

extern "C" fm_status fm_set_gemm_splitk(int enable) {
  if (enable != 0 && enable != 1)
    return fail(FM_ERR_INVALID_ARG, "fm_set_gemm_splitk: enable must be 0 or 1");
  g_gemm_splitk.store(enable, std::memory_order_relaxed);
  return FM_OK;
}

// the small-grid path would split this GEMM (the workspace must hold M x N int32)
static bool gemm_would_split(long long M, long long N, long long K) {
  if (!g_gemm_splitk.load(std::memory_order_relaxed)) return false;
  const int sms = sm_count();
  const long long mt = (M + kGemmBM - 1) / kGemmBM;
  if (K % kGemmBK || mt * ((N + 127) / 128) >= sms) return false;
  const int BN = mt * ((N + 63) / 64) < sms ? 32 : 64;
  int kbs = 0;
  return gemm_splits(M, N, K, BN, sms, &kbs) > 1;
}

template <int BN, int STAGES, int AR = kGemmBM>
static fm_status launch_gemm_t(const CUtensorMap &ta, const CUtensorMap &tb, long long M,
                               long long N, long long K, GemmEpilogue ep, int32_t *split_ws,
                               cudaStream_t s) {
  constexpr int smem = gemm_smem_bytes(BN, STAGES, AR);
  static_assert(smem <= 227 * 1024, "shared memory per CTA");
  const int nkb = (int)(K / kGemmBK);
  int kbs = nkb, splits = 1;
  if (split_ws && g_gemm_splitk.load(std::memory_order_relaxed))
    splits = gemm_splits(M, N, K, BN, sm_count(), &kbs);
  auto kern = splits > 1 ? k_gemm_i8_tc<BN, STAGES, true, AR> : k_gemm_i8_tc<BN, STAGES, false, AR>;
  FM_CHECK_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  if (splits > 1) {
    ep.split_acc = split_ws;
    FM_CHECK_CUDA(cudaMemsetAsync(split_ws, 0, sizeof(int32_t) * (size_t)(M * N), s));
  }
  dim3 grid((unsigned)((N + BN - 1) / BN), (unsigned)((M + kGemmBM - 1) / kGemmBM),
            (unsigned)splits);
  FM_TRY(launch_ex("k_gemm_i8_tc", kern, grid, kGemmThreads, smem, s, ta, tb, nkb, kbs, ep));
  FM_TRY(launched("k_gemm_i8_tc"));
  if (splits > 1) {
    const long long n = M * ((N + 31) / 32);
    FM_TRY(launch_ex("k_gemm_splitk_epilogue", k_gemm_splitk_epilogue, (unsigned)((n + 127) / 128),
                     128, 0, s, ep));
    FM_TRY(launched("k_gemm_splitk_epilogue"));
  }
  return FM_OK;
}

// Split K over a thread-block cluster (k_gemm_i8_cl), for a decode batch
// whose 32-wide tiles are fewer than the SMs: S ranks per tile, chosen so that
// the grid covers about two CTAs per SM and every rank gets a K block.
// Process-wide, off by default: measured slower on the 2.7B decode out_proj
// (20.4 against 17.7 us per launch; the step 6.90 against 6.75 ms).
static std::atomic<int> g_gemm_cluster{0};

extern "C" fm_status fm_set_gemm_cluster(int enable) {
  if (enable != 0 && enable != 1)
    return fail(FM_ERR_INVALID_ARG, "fm_set_gemm_cluster: %d is not 0 or 1", enable);
  g_gemm_cluster.store(enable, std::memory_order_relaxed);
  return FM_OK;
}

static int gemm_cluster_ranks(long long N, long long K, int sms) {
  const long long tiles = (N + 31) / 32, nkb = K / kGemmBK;
  int S = (int)((2LL * sms + tiles - 1) / tiles);
  if (S > 8) S = 8;
  while (S >= 2 && (long long)(S - 1) * ((nkb + S - 1) / S) >= nkb) --S;
  return S;
}

template <int S>
static fm_status launch_gemm_cl_t(const CUtensorMap &ta, const CUtensorMap &tb, long long N,
                                  long long K, const GemmEpilogue &ep, cudaStream_t s) {
  constexpr int BN = 32, STAGES = 4;
  constexpr int smem = gemm_cl_smem_bytes(BN, STAGES);
  static_assert(smem <= 75 * 1024, "three cluster CTAs per SM");
  auto kern = k_gemm_i8_cl<BN, STAGES, S>;
  FM_CHECK_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  const int nkb = (int)(K / kGemmBK);
  const int per = (nkb + S - 1) / S;
  cudaLaunchConfig_t cfg = {};  // no attributes unless set below
  cfg.gridDim = dim3((unsigned)((N + BN - 1) / BN), 1, S);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = S;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g_pdl.load(std::memory_order_relaxed) ? 2 : 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ta, tb, nkb, per, ep);
  if (e != cudaSuccess)
    return fail(FM_ERR_CUDA, "launch of k_gemm_i8_cl: %s", cudaGetErrorString(e));
  return launched("k_gemm_i8_cl");
}

template <int BN, int STAGES, int EW>
static fm_status launch_gemm_persist(const CUtensorMap &ta, const CUtensorMap &tb, long long M,
                                     long long N, long long K, int sms, GemmEpilogue ep,
                                     cudaStream_t s) {
  CUtensorMap to[3];
  FM_TRY(gemm_output_maps(ep, to, ta));
  constexpr int smem = PersistSmem<BN, STAGES, EW>::kBytes;
  static_assert(smem <= 227 * 1024, "shared memory per CTA");
  auto kern = k_gemm_i8_persist<BN, STAGES, EW>;
  FM_CHECK_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  const int m_tiles = (int)((M + kGemmBM - 1) / kGemmBM), n_tiles = (int)((N + BN - 1) / BN);
  const long long tiles = (long long)m_tiles * n_tiles;
  const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);
  FM_TRY(launch_ex("k_gemm_i8_persist", kern, grid, 64 + 32 * EW, smem, s, ta, tb, to[0], to[1],
                   to[2], (int)(K / kGemmBK), m_tiles, n_tiles, ep));
  return launched("k_gemm_i8_persist");
}

static int sm_count() {
  constexpr int kMaxDevices = 64;
  static std::atomic<int> cache[kMaxDevices];  // zero-initialised (static storage)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (!n) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Large problems: the persistent kernel, 128 x 256 tiles when there are at
// least two per SM (fewer L2 bytes per MMA), else 128 x 128.  Small grids
// (fewer 128-wide tiles than SMs, e.g. out_proj at 130M shapes or a decode
// batch): one 128 x 64 tile per CTA (128 x 32 when even those are fewer than
// the SMs), two CTAs per SM.
// split_ws (nullable, M x N int32): lets the small-grid path split K.
// Tile width of the persistent GEMM, process-wide: 0 (default) chooses by the
// grid (256 when there are at least two 256-wide tiles per SM), 128 or 256
// forces that width wherever the persistent kernel runs (tuning).
static std::atomic<int> g_gemm_tile{0};

extern "C" fm_status fm_set_gemm_tile(int bn) {
  if (bn != 0 && bn != 128 && bn != 256)
    return fail(FM_ERR_INVALID_ARG, "fm_set_gemm_tile: %d is not 0, 128 or 256", bn);
  g_gemm_tile.store(bn, std::memory_order_relaxed);
  return FM_OK;
}

static fm_status launch_gemm(const int8_t *A, long long M, const int8_t *W, long long N,
                             long long K, const GemmEpilogue &ep, cudaStream_t s,
                             int32_t *split_ws = nullptr) {
  if (K % kGemmBK) return fail(FM_ERR_SHAPE, "gemm: K=%lld is not a multiple of 128", K);
  if ((M + kGemmBM - 1) / kGemmBM > 65535 || (N + 63) / 64 > 65535)
    return fail(FM_ERR_SHAPE, "gemm: M=%lld or N=%lld too large", M, N);
  CUtensorMap ta, tb;
  const long long mt = (M + kGemmBM - 1) / kGemmBM;
  const long long tiles256 = mt * ((N + 255) / 256), tiles128 = mt * ((N + 127) / 128);
  const int sms = sm_count();
  FM_TRY(make_tmap(&ta, A, M, K, kGemmBM));
  const int force = g_gemm_tile.load(std::memory_order_relaxed);
  const bool persist = tiles256 >= 2LL * sms || tiles128 >= sms;
  if (persist && (force == 256 || (force == 0 && tiles256 >= 2LL * sms))) {
    FM_TRY(make_tmap(&tb, W, N, K, 256));
    return launch_gemm_persist<256, 3, 8>(ta, tb, M, N, K, sms, ep, s);
  }
  if (persist) {
    FM_TRY(make_tmap(&tb, W, N, K, 128));
    return launch_gemm_persist<128, 5, 8>(ta, tb, M, N, K, sms, ep, s);
  }
  const bool narrow = mt * ((N + 63) / 64) < sms;  // fewer 64-wide tiles than SMs: 32 wide
  FM_TRY(make_tmap(&tb, W, N, K, narrow ? 32 : 64));
  if (M <= 64) {
    // a decode batch: only the 64 real rows of A per stage, so the weight
    // stream gets a deeper ring (64 wide: 6 x 16 KB, two CTAs per SM; 32 wide,
    // fewer CTAs than SMs: 16 x 12 KB, one per SM)
    FM_TRY(make_tmap(&ta, A, M, K, 64));
    if (narrow && g_gemm_cluster.load(std::memory_order_relaxed) &&
        !(split_ws && g_gemm_splitk.load(std::memory_order_relaxed))) {
      switch (gemm_cluster_ranks(N, K, sms)) {
        case 2: return launch_gemm_cl_t<2>(ta, tb, N, K, ep, s);
        case 3: return launch_gemm_cl_t<3>(ta, tb, N, K, ep, s);
        case 4: return launch_gemm_cl_t<4>(ta, tb, N, K, ep, s);
        case 5: return launch_gemm_cl_t<5>(ta, tb, N, K, ep, s);
        case 6: return launch_gemm_cl_t<6>(ta, tb, N, K, ep, s);
        case 7: return launch_gemm_cl_t<7>(ta, tb, N, K, ep, s);
        case 8: return launch_gemm_cl_t<8>(ta, tb, N, K, ep, s);
        default: break;  // too few K blocks to split
      }
    }
    if (narrow) return launch_gemm_t<32, 16, 64>(ta, tb, M, N, K, ep, split_ws, s);
    return launch_gemm_t<64, 6, 64>(ta, tb, M, N, K, ep, split_ws, s);
  }
  if (narrow) return launch_gemm_t<32, 6>(ta, tb, M, N, K, ep, split_ws, s);
  return launch_gemm_t<64, 4>(ta, tb, M, N, K, ep, split_ws, s);
}

static fm_status launch_hadamard_quant(const float *x, long long M, int K, const float *prenorm_w,
                                       int rotate, int mode, const float *static_amax, int8_t *q,
                                       float *s_x, float *amax_row, cudaStream_t s) {
  if (M <= 0) return FM_OK;

  // two 256-blocks per warp when they pair up and there are rows enough to
  // fill the GPU; a handful of rows (a decode batch) keeps one per warp
  const int nb = K / 256;
  if (nb % 2 == 0 && M >= 2LL * sm_count())
    FM_TRY(launch_ex("k_hadamard_quant", k_hadamard_quant<2>, (unsigned)M, 32 * (nb / 2), 0, s, x,
                     K, prenorm_w, rotate, mode, static_amax, q, s_x, amax_row));
  else
    FM_TRY(launch_ex("k_hadamard_quant", k_hadamard_quant<1>, (unsigned)M, 32 * nb, 0, s, x, K,
                     prenorm_w, rotate, mode, static_amax, q, s_x, amax_row));
  return launched("k_hadamard_quant");
}

static fm_status launch_conv(const int8_t *u, int B, int T, int cc, const int8_t *wq,
                             const int32_t *bq, const int32_t *exps, int8_t *conv_state,
                             int8_t *out, unsigned int *amax, cudaStream_t s,
                             int32_t *e_tok = nullptr, const Dims *d = nullptr) {
  if ((long long)B * T == 0) return FM_OK;
  const int groups = (cc / kConvCPT + kConvQuads - 1) / kConvQuads;
  if (B > 65535) return fail(FM_ERR_SHAPE, "conv: B too large");
  if (e_tok && (!d || amax)) return fail(FM_ERR_INVALID_ARG, "conv: per-token exponents misused");
  const int di = d ? d->di : 0, hd = d ? d->hd : 0, ds = d ? d->ds : 0;
  if (T >= kConvTT) {
    const unsigned tiles = (unsigned)((T + kConvTokens - 1) / kConvTokens);
    const dim3 grid(tiles, groups, B);
    auto kern = e_tok ? k_conv1d_pot<kConvTT, kConvTG, true>
                      : (amax ? k_conv1d_pot<kConvTT, kConvTG, false, true>
                              : k_conv1d_pot<kConvTT, kConvTG, false, false>);
    FM_TRY(launch_ex("k_conv1d_pot", kern, grid, kConvQuads * kConvTG, 0, s, u, T, cc, wq, bq,
                     exps, conv_state, out, amax, nullptr, e_tok, di, hd, ds));
  } else {  // decode steps and short chunks: one token per thread
    const dim3 grid((unsigned)T, groups, B);
    int8_t *state_out = T == 1 ? conv_state : nullptr;
    auto kern = e_tok ? k_conv1d_pot<1, 1, true>
                      : (amax ? k_conv1d_pot<1, 1, false, true> : k_conv1d_pot<1, 1, false, false>);
    FM_TRY(launch_ex("k_conv1d_pot", kern, grid, kConvQuads, 0, s, u, T, cc, wq, bq, exps,
                     conv_state, out, amax, state_out, e_tok, di, hd, ds));
  }
  FM_TRY(launched("k_conv1d_pot"));
  if (conv_state && T > 1) {  // a single step updates its state in the conv kernel
    const long long n = (long long)B * cc;
    FM_TRY(launch_ex("k_conv_state_update", k_conv_state_update, (unsigned)((n + 255) / 256), 256,
                     0, s, u, B, T, cc, conv_state));
    FM_TRY(launched("k_conv_state_update"));
  }
  return FM_OK;
}

// The state spec, process-wide: the word width and the increment's guard
// bits.  (31, 0) is the method as built; (16, 7) the narrow state whose
// increment is rounded after the u B product (u with 7 guard bits).
static std::atomic<int> g_state_bits{31};
static std::atomic<int> g_state_guard{0};

extern "C" fm_status fm_set_state_spec(int bits, int guard) {
  if (!((bits == 31 && guard == 0) || (bits == 16 && guard == 7)))
    return fail(FM_ERR_INVALID_ARG, "fm_set_state_spec: (%d, %d) is not a supported spec "
                "(31, 0) or (16, 7)", bits, guard);
  g_state_bits.store(bits, std::memory_order_relaxed);
  g_state_guard.store(guard, std::memory_order_relaxed);
  return FM_OK;
}
static bool state16() { return g_state_bits.load(std::memory_order_relaxed) == 16; }

// Conv-output exponent granularity, process-wide: 0 (default) the static
// per-head / B / C exponents as built, 1 per token (the conv requantises each
// token's groups at their own power-of-two exponent; the scans shift by them).
static std::atomic<int> g_xbc_tok{0};

extern "C" fm_status fm_set_xbc_exponents(int per_token) {
  if (per_token != 0 && per_token != 1)
    return fail(FM_ERR_INVALID_ARG, "fm_set_xbc_exponents: per_token must be 0 or 1");
  g_xbc_tok.store(per_token, std::memory_order_relaxed);
  return FM_OK;
}
static bool xbc_tok() { return g_xbc_tok.load(std::memory_order_relaxed) == 1; }

static ScanArgs scan_args(const Dims &d, const int8_t *xbc, const float *dt_raw, int T,
                          const float *dt_bias, const int32_t *A_q, const int32_t *D_q,
                          const int32_t *exps, const fm_exp_layout &X, int32_t *state, int32_t *y,
                          unsigned long long *stat, const int32_t *e_tok = nullptr) {
  ScanArgs a;
  a.xbc = xbc;
  a.dt_raw = dt_raw;
  a.T = T;
  a.nh = d.nh;
  a.hd = d.hd;
  a.cc = d.cc;
  a.di = d.di;
  a.dt_bias = dt_bias;
  a.A_q = A_q;
  a.D_q = D_q;
  a.e_x = exps + X.e_x;
  a.e_B = exps + X.e_B;
  a.e_C = exps + X.e_C;
  a.e_h = exps + X.e_h;
  a.e_y = exps + X.e_y;
  a.e_D = exps + X.e_D;
  a.state = state;
  a.y = y;
  a.stat = stat;
  a.hlim = state16() ? kH16Lim : (int)kHLim;
  a.guard = g_state_guard.load(std::memory_order_relaxed);
  a.e_tok = e_tok;
  return a;
}

template <int MODE>
static fm_status launch_scan(const ScanArgs &a, int B, cudaStream_t s) {
  if ((long long)B * a.T == 0) return FM_OK;
  if (B > 65535) return fail(FM_ERR_SHAPE, "scan: B too large");
  dim3 grid(a.hd / kScanPC, a.nh, B);
  k_ssm_scan_pot<MODE><<<grid, kScanThreads, 0, s>>>(a);
  return launched("k_ssm_scan_pot");
}

// Sequential-scan tile (n per thread, p per CTA, steps per staged chunk);
// process-wide, chosen with fm_set_scan_tile among the compiled variants.
struct ScanTile {
  int npt, pc, tch;
};
// (4, 0, 32) first: the default, 32-step chunks with the channels per CTA
// chosen by the grid (pc = 0): 8 where there are at least three such CTAs per
// SM, else 4.  Measured: 32-step chunks against 16, 130M stack 7.10 -> 6.74 ms
// per step, 2.7B stack 195.4 -> 191.7 ms (the per-chunk work -- the barrier
// wait, the growth-bound test, the slot release, the output epilogue -- is
// spread over twice the steps, and the epilogue uses all 32 lanes); 8 channels
// per CTA against 4 at 2.7B 191.7 -> 185.3 ms (twice the warps per SM, B and C
// staged once for 8 channels), at 130M B = 1 8.02 against 6.76 ms (too few CTAs).
static const ScanTile kScanTiles[] = {{4, 0, 32}, {4, 4, 32}, {4, 8, 32}, {4, 4, 16},
                                      {4, 2, 16}, {4, 8, 16}, {8, 4, 16}, {8, 2, 16},
                                      {8, 8, 16}};
static std::atomic<int> g_scan_tile{0};
// 0: the sequential fixed-point scan (the method); 1: the chunked scan mode for
// prefills of more than one token (single steps stay sequential)
static std::atomic<int> g_scan_mode{0};

extern "C" fm_status fm_set_scan_mode(int mode) {
  if (mode != 0 && mode != 1) return fail(FM_ERR_INVALID_ARG, "fm_set_scan_mode: bad mode %d", mode);
  g_scan_mode.store(mode, std::memory_order_relaxed);
  return FM_OK;
}
static bool use_ssd(int T) { return T > 1 && g_scan_mode.load(std::memory_order_relaxed) == 1; }
static ScanTile scan_tile() { return kScanTiles[g_scan_tile.load(std::memory_order_relaxed)]; }
// Set while this thread queues the runs of a pipelined stack prefill
// (fm_stack_prefill): on a grid too small for 8 channels per CTA the default
// tile then stages 16-step chunks, half the shared memory of 32, so that more
// CTAs of the neighbouring runs' kernels fit beside the scan.  Measured, 130M
// stack at B = 1: 4 runs with 16-step chunks 340.3 k tokens/s, with 32-step
// chunks 332.2 k (2 runs: 323.9 k and 335.7 k).
static thread_local bool t_pipelined_run = false;

extern "C" fm_status fm_set_scan_tile(int npt, int pc, int tch) {
  for (int i = 0; i < (int)(sizeof(kScanTiles) / sizeof(kScanTiles[0])); ++i)
    if (kScanTiles[i].npt == npt && kScanTiles[i].pc == pc && kScanTiles[i].tch == tch) {
      g_scan_tile.store(i, std::memory_order_relaxed);
      return FM_OK;
    }
  return fail(FM_ERR_INVALID_ARG, "fm_set_scan_tile: (%d, %d, %d) is not a compiled variant", npt,
              pc, tch);
}

template <int NPT, int PC, int TCH, bool S16, bool TOK>
static fm_status launch_seq(const ScanSeqArgs &a, int B, cudaStream_t s) {
  using Sm = ScanSeqSmem<NPT, PC, TCH>;
  constexpr int smem = (int)sizeof(Sm);
  auto kern = k_scan_seq<NPT, PC, TCH, S16, TOK>;
  FM_CHECK_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  dim3 grid(a.hd / PC, a.nh, B);
  FM_TRY(launch_ex("k_scan_seq", kern, grid, PC * (128 / NPT) + 32, smem, s, a));
  return launched("k_scan_seq");
}

struct ScanWs {
  int32_t *dA;  // [B, nh, Tp]
  int32_t *u;   // [B, nh, hd, Tp]
  int8_t *xs;   // [B, nh, hd, Tp]: x codes
  int32_t *bc;  // [B*T, 256]
  long long *bound;  // [B, nh, Tp/16, hd]
  int32_t *osh;      // [B, nh, Tp] per-token output shifts (per-token exponents only)
};

// prep (parallel over token tiles and heads) + the sequential kernel
static fm_status launch_scan_v2(const ScanArgs &a, int B, const ScanWs &w, cudaStream_t s) {
  const long long M = (long long)B * a.T;
  if (M == 0) return FM_OK;
  if (B > 65535 || M > 2147483647LL) return fail(FM_ERR_SHAPE, "scan: B or B*T too large");
  if (a.T == 1) {  // decode: one step per sequence, no staging
    // the step kernel takes the spec's clamp and guard bits as constants
    const bool narrow = a.hlim <= kH16Lim;
    if (narrow ? (a.hlim != kH16Lim || a.guard != kH16Guard) : (a.hlim != kHLim || a.guard != 0))
      return fail(FM_ERR_INVALID_ARG, "scan step: state spec (%d, %d) is not a supported one",
                  a.hlim, a.guard);
    if (narrow)
      FM_TRY(launch_ex("k_scan_step", k_scan_step<true>, dim3(a.nh, B), 256, 0, s, a));
    else
      FM_TRY(launch_ex("k_scan_step", k_scan_step<false>, dim3(a.nh, B), 256, 0, s, a));
    return launched("k_scan_step");
  }
  const long long Tp = scan_tpad(a.T);
  ScanPrepArgs p;
  p.xbc = a.xbc;
  p.dt_raw = a.dt_raw;
  p.T = a.T;
  p.nh = a.nh;
  p.hd = a.hd;
  p.cc = a.cc;
  p.di = a.di;
  p.dt_bias = a.dt_bias;
  p.A_q = a.A_q;
  p.D_q = a.D_q;
  p.e_x = a.e_x;
  p.e_B = a.e_B;
  p.e_h = a.e_h;
  p.e_y = a.e_y;
  p.e_D = a.e_D;
  p.dA = w.dA;
  p.u = w.u;
  p.xs = w.xs;
  p.bc = w.bc;
  p.bound = w.bound;
  p.guard = a.guard;
  p.e_tok = a.e_tok;
  p.osh = a.e_tok ? w.osh : nullptr;
  if (a.e_tok && !w.osh) return fail(FM_ERR_WORKSPACE, "scan: per-token shifts need workspace");
  if (p.e_tok)
    FM_TRY(launch_ex("k_scan_prep", k_scan_prep<true>, dim3((unsigned)(Tp / kPrepTT), a.nh, B),
                     256, 0, s, p));
  else
    FM_TRY(launch_ex("k_scan_prep", k_scan_prep<false>, dim3((unsigned)(Tp / kPrepTT), a.nh, B),
                     256, 0, s, p));
  FM_TRY(launched("k_scan_prep"));
  ScanSeqArgs q;
  q.dA = w.dA;
  q.u = w.u;
  q.xs = w.xs;
  q.D_q = a.D_q;
  q.e_x = a.e_x;
  q.e_D = a.e_D;
  q.bc = w.bc;
  q.bound = w.bound;
  q.T = a.T;
  q.nh = a.nh;
  q.hd = a.hd;
  q.di = a.di;
  q.e_C = a.e_C;
  q.e_h = a.e_h;
  q.e_y = a.e_y;
  q.state = a.state;
  q.y = a.y;
  q.osh = p.osh;
  ScanTile t = scan_tile();
  if (t.pc == 0) {
    t.pc = (long long)B * a.nh * a.hd / 8 >= 3LL * sm_count() ? 8 : 4;
    if (t_pipelined_run && t.pc == 4) t.tch = 16;
  }
#define FM_SEQ(N, P, C)                                                          \
  if (t.npt == N && t.pc == P && t.tch == C) {                                   \
    if (q.osh)                                                                   \
      return state16() ? launch_seq<N, P, C, true, true>(q, B, s)                \
                       : launch_seq<N, P, C, false, true>(q, B, s);              \
    return state16() ? launch_seq<N, P, C, true, false>(q, B, s)                 \
                     : launch_seq<N, P, C, false, false>(q, B, s);               \
  }
  FM_SEQ(4, 4, 16)
  FM_SEQ(4, 2, 16)
  FM_SEQ(4, 8, 16)
  FM_SEQ(8, 4, 16)
  FM_SEQ(8, 2, 16)
  FM_SEQ(8, 8, 16)
  FM_SEQ(4, 4, 32)
  FM_SEQ(4, 8, 32)
#undef FM_SEQ
  return fail(FM_ERR_INVALID_ARG, "scan tile (%d, %d, %d) is not compiled", t.npt, t.pc, t.tch);
}

// ------------------------------------------------------------------ entry points
extern "C" fm_status fm_hadamard_quant(const float *x, int64_t M, int64_t K, const float *prenorm_w,
                                       int rotate, int mode, const float *static_amax, int8_t *q,
                                       float *s_x, float *amax_row, fm_stream stream) {
  if (M < 0) return fail(FM_ERR_SHAPE, "fm_hadamard_quant: M < 0");
  if (K <= 0 || K % 256 || K > 256 * kMaxBlocks)
    return fail(FM_ERR_SHAPE, "fm_hadamard_quant: K=%lld must be a multiple of 256 <= %d",
                (long long)K, 256 * kMaxBlocks);
  if (M > 2147483647LL) return fail(FM_ERR_SHAPE, "fm_hadamard_quant: M too large");
  if (mode != FM_DYNAMIC && mode != FM_STATIC)
    return fail(FM_ERR_INVALID_ARG, "fm_hadamard_quant: bad mode %d", mode);
  if (M == 0) return FM_OK;
  NEED(x);
  NEED(q);
  NEED(s_x);
  OPT(prenorm_w);
  OPT(amax_row);
  if (mode == FM_STATIC && !static_amax)
    return fail(FM_ERR_INVALID_ARG, "fm_hadamard_quant: static mode needs static_amax");
  return launch_hadamard_quant(x, M, (int)K, prenorm_w, rotate ? 1 : 0, mode, static_amax, q, s_x,
                               amax_row, (cudaStream_t)stream);
}

extern "C" fm_status fm_prepare_linear(const float *W, int64_t N, int64_t K, int rotate,
                                       int8_t *Wq, float *s_w, fm_stream stream) {
  if (N < 0 || N > 2147483647LL) return fail(FM_ERR_SHAPE, "fm_prepare_linear: bad N");
  if (K <= 0 || K % 256 || K > 256 * kMaxBlocks)
    return fail(FM_ERR_SHAPE, "fm_prepare_linear: K=%lld must be a multiple of 256", (long long)K);
  if (N == 0) return FM_OK;
  NEED(W);
  NEED(Wq);
  NEED(s_w);
  k_prepare_linear<<<(unsigned)N, 32 * (int)(K / 256), 0, (cudaStream_t)stream>>>(
      W, (int)K, rotate ? 1 : 0, Wq, s_w);
  return launched("k_prepare_linear");
}

static GemmEpilogue plain_epilogue(long long M, long long N, const float *s_x, const float *s_w,
                                   const float *residual, float *Y, int32_t *acc_out) {
  GemmEpilogue ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.mode = 0;
  ep.M = M;
  ep.N = N;
  ep.s_x = s_x;
  ep.s_w = s_w;
  ep.residual = residual;
  ep.Y = Y;
  ep.acc_out = acc_out;
  return ep;
}

extern "C" fm_status fm_w8a8_gemm(const int8_t *A, const float *s_x, int64_t M, const int8_t *Wq,
                                  const float *s_w, int64_t N, int64_t K, const float *residual,
                                  float *Y, int32_t *acc_out, fm_stream stream) {
  if (M < 0 || N < 0 || K <= 0 || K % 128)
    return fail(FM_ERR_SHAPE, "fm_w8a8_gemm: need M, N >= 0 and K a positive multiple of 128");
  if (M == 0 || N == 0) return FM_OK;
  NEED(A);
  NEED(s_x);
  NEED(Wq);
  NEED(s_w);
  NEED(Y);
  OPT(residual);
  OPT(acc_out);
  return launch_gemm(A, M, Wq, N, K, plain_epilogue(M, N, s_x, s_w, residual, Y, acc_out),
                     (cudaStream_t)stream);
}

static fm_status in_proj_impl(const int8_t *A, const float *s_x, long long M, const int8_t *Wq,
                              const float *s_w, const Dims &d, const int32_t *e_u, float *z,
                              int8_t *xbc, float *dt, cudaStream_t s,
                              int32_t *split_ws = nullptr) {
  GemmEpilogue ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.mode = 1;
  ep.M = M;
  ep.N = d.n_in;
  ep.s_x = s_x;
  ep.s_w = s_w;
  ep.di = d.di;
  ep.cc = d.cc;
  ep.nh = d.nh;
  ep.e_u = e_u;
  ep.z = z;
  ep.xbc = xbc;
  ep.dt = dt;
  return launch_gemm(A, M, Wq, d.n_in, d.dm, ep, s, split_ws);
}

extern "C" fm_status fm_in_proj(const int8_t *A, const float *s_x, int64_t M, const int8_t *Wq,
                                const float *s_w, const fm_shape *shape, const int32_t *exps,
                                float *z, int8_t *xbc, float *dt, fm_stream stream) {
  Dims d;
  FM_TRY(check_shape(shape, &d, __func__));
  if (M < 0) return fail(FM_ERR_SHAPE, "fm_in_proj: M < 0");
  if (M == 0) return FM_OK;
  NEED(A);
  NEED(s_x);
  NEED(Wq);
  NEED(s_w);
  NEED(exps);
  NEED(z);
  NEED(xbc);
  NEED(dt);
  return in_proj_impl(A, s_x, M, Wq, s_w, d, exps, z, xbc, dt, (cudaStream_t)stream);
}

extern "C" size_t fm_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  return gemm_would_split(M, N, K) ? sizeof(int32_t) * (size_t)(M * N) : 0;
}

static fm_status gemm_ws(void *ws, size_t ws_bytes, long long M, long long N, long long K,
                         int32_t **split, const char *fn) {
  const size_t need = fm_gemm_workspace_bytes(M, N, K);
  *split = nullptr;
  if (!need) return FM_OK;
  if (!ws || ws_bytes < need || !aligned16(ws))
    return fail(FM_ERR_WORKSPACE, "%s: workspace needs %zu bytes", fn, need);
  *split = reinterpret_cast<int32_t *>(ws);
  return FM_OK;
}

extern "C" fm_status fm_w8a8_gemm_ws(const int8_t *A, const float *s_x, int64_t M,
                                     const int8_t *Wq, const float *s_w, int64_t N, int64_t K,
                                     const float *residual, float *Y, int32_t *acc_out, void *ws,
                                     size_t ws_bytes, fm_stream stream) {
  if (M < 0 || N < 0 || K <= 0 || K % 128)
    return fail(FM_ERR_SHAPE, "fm_w8a8_gemm_ws: need M, N >= 0 and K a positive multiple of 128");
  if (M == 0 || N == 0) return FM_OK;
  NEED(A);
  NEED(s_x);
  NEED(Wq);
  NEED(s_w);
  NEED(Y);
  OPT(residual);
  OPT(acc_out);
  int32_t *split = nullptr;
  FM_TRY(gemm_ws(ws, ws_bytes, M, N, K, &split, __func__));
  return launch_gemm(A, M, Wq, N, K, plain_epilogue(M, N, s_x, s_w, residual, Y, acc_out),
                     (cudaStream_t)stream, split);
}

extern "C" fm_status fm_in_proj_ws(const int8_t *A, const float *s_x, int64_t M,
                                   const int8_t *Wq, const float *s_w, const fm_shape *shape,
                                   const int32_t *exps, float *z, int8_t *xbc, float *dt,
                                   void *ws, size_t ws_bytes, fm_stream stream) {
  Dims d;
  FM_TRY(check_shape(shape, &d, __func__));
  if (M < 0) return fail(FM_ERR_SHAPE, "fm_in_proj_ws: M < 0");
  if (M == 0) return FM_OK;
  NEED(A);
  NEED(s_x);
  NEED(Wq);
  NEED(s_w);
  NEED(exps);
  NEED(z);
  NEED(xbc);
  NEED(dt);
  int32_t *split = nullptr;
  FM_TRY(gemm_ws(ws, ws_bytes, M, d.n_in, d.dm, &split, __func__));
  return in_proj_impl(A, s_x, M, Wq, s_w, d, exps, z, xbc, dt, (cudaStream_t)stream, split);
}

extern "C" fm_status fm_conv1d_pot(const int8_t *u, int B, int T, const fm_shape *shape,
                                   const int8_t *wq, const int32_t *bq, const int32_t *exps,
                                   int8_t *conv_state, int8_t *out, fm_stream stream) {
  Dims d;
  FM_TRY(check_shape(shape, &d, __func__));
  if (B < 0 || T < 0) return fail(FM_ERR_SHAPE, "fm_conv1d_pot: B, T must be >= 0");
  if ((long long)B * T == 0) return FM_OK;
  NEED(u);
  NEED(wq);
  NEED(bq);
  NEED(exps);
  NEED(out);
  OPT(conv_state);
  return launch_conv(u, B, T, d.cc, wq, bq, exps, conv_state, out, nullptr, (cudaStream_t)stream);
}

extern "C" fm_status fm_conv1d_pot_tok(const int8_t *u, int B, int T, const fm_shape *shape,
                                       const int8_t *wq, const int32_t *bq, const int32_t *exps,
                                       int8_t *conv_state, int8_t *out, int32_t *e_tok,
                                       fm_stream stream) {
  Dims d;
  FM_TRY(check_shape(shape, &d, __func__));
  if (B < 0 || T < 0) return fail(FM_ERR_SHAPE, "fm_conv1d_pot_tok: B, T must be >= 0");
  if ((long long)B * T == 0) return FM_OK;
  NEED(u);
  NEED(wq);
  NEED(bq);
  NEED(exps);
  NEED(out);
  NEED(e_tok);
  OPT(conv_state);
  return launch_conv(u, B, T, d.cc, wq, bq, exps, conv_state, out, nullptr, (cudaStream_t)stream,
                     e_tok, &d);
}

namespace {
struct Carver {
  uint8_t *base;
  size_t off;
  template <typename T>
  T *take(size_t n) {
    off = (off + 255) & ~size_t(255);
    T *p = base ? reinterpret_cast<T *>(base + off) : nullptr;
    off += n * sizeof(T);
    return p;
  }
};

ScanWs carve_scan(Carver &c, const Dims &d, int B, int T, bool tok) {
  ScanWs w;
  w.osh = nullptr;
  if (T == 1) {  // single steps run k_scan_step, which stages nothing
    w.dA = nullptr;
    w.u = w.bc = nullptr;
    w.xs = nullptr;
    w.bound = nullptr;
    return w;
  }
  const long long Tp = scan_tpad(T), M = (long long)B * T;
  w.dA = c.take<int32_t>((long long)B * d.nh * Tp);
  w.u = c.take<int32_t>((long long)B * d.di * Tp);
  w.xs = c.take<int8_t>((long long)B * d.di * Tp);
  w.bc = c.take<int32_t>(M * 256);
  w.bound = c.take<long long>((long long)B * d.di * (Tp / 16));
  if (tok) w.osh = c.take<int32_t>((long long)B * d.nh * Tp);
  return w;
}
}  // namespace

static size_t scan_ws_bytes(const fm_shape *shape, int B, int T, bool tok) {
  Dims d;
  if (check_shape(shape, &d, "fm_scan_workspace_bytes") != FM_OK || B < 0 || T < 0) return 0;
  Carver c{nullptr, 0};
  carve_scan(c, d, B, T, tok);
  return c.off + 256;
}
extern "C" size_t fm_scan_workspace_bytes(const fm_shape *shape, int B, int T) {
  return scan_ws_bytes(shape, B, T, false);
}
extern "C" size_t fm_scan_workspace_bytes_tok(const fm_shape *shape, int B, int T) {
  return scan_ws_bytes(shape, B, T, true);
}

extern "C" fm_status fm_ssm_scan_pot(const int8_t *xbc, const float *dt_raw, int B, int T,
                                     const fm_shape *shape, const float *dt_bias,
                                     const int32_t *A_q, const int32_t *D_q, const int32_t *exps,
                                     int32_t *state, int32_t *y, void *ws, size_t ws_bytes,
                                     fm_stream stream) {
  Dims d;
  FM_TRY(check_shape(shape, &d, __func__));
  if (B < 0 || T < 0) return fail(FM_ERR_SHAPE, "fm_ssm_scan_pot: B, T must be >= 0");
  if ((long long)B * T == 0) return FM_OK;
  NEED(xbc);
  NEED(dt_raw);
  NEED(dt_bias);
  NEED(A_q);
  NEED(D_q);
  NEED(exps);
  NEED(y);
  OPT(state);
  const size_t need = fm_scan_workspace_bytes(shape, B, T);
  if (!ws || ws_bytes < need || !aligned16(ws))
    return fail(FM_ERR_WORKSPACE, "fm_ssm_scan_pot: workspace needs %zu bytes", need);
  Carver c{reinterpret_cast<uint8_t *>(ws), 0};
  const ScanWs w = carve_scan(c, d, B, T, false);
  const fm_exp_layout X = fm_exp_table_layout(shape);
  return launch_scan_v2(scan_args(d, xbc, dt_raw, T, dt_bias, A_q, D_q, exps, X, state, y, nullptr),
                        B, w, (cudaStream_t)stream);
}

extern "C" fm_status fm_ssm_scan_pot_tok(const int8_t *xbc, const float *dt_raw, int B, int T,
                                         const fm_shape *shape, const float *dt_bias,
                                         const int32_t *A_q, const int32_t *D_q,
                                         const int32_t *exps, const int32_t *e_tok,
                                         int32_t *state, int32_t *y, void *ws, size_t ws_bytes,
                                         fm_stream stream) {
  Dims d;
  FM_TRY(check_shape(shape, &d, __func__));
  if (B < 0 || T < 0) return fail(FM_ERR_SHAPE, "fm_ssm_scan_pot_tok: B, T must be >= 0");
  if ((long long)B * T == 0) return FM_OK;
  NEED(xbc);
  NEED(dt_raw);
  NEED(dt_bias);
  NEED(A_q);
  NEED(D_q);
  NEED(exps);
  NEED(e_tok);
  NEED(y);
  OPT(state);
  const size_t need = fm_scan_workspace_bytes_tok(shape, B, T);
  if (!ws || ws_bytes < need || !aligned16(ws))
    return fail(FM_ERR_WORKSPACE, "fm_ssm_scan_pot_tok: workspace needs %zu bytes", need);
  Carver c{reinterpret_cast<uint8_t *>(ws), 0};
  const ScanWs w = carve_scan(c, d, B, T, true);
  const fm_exp_layout X = fm_exp_table_layout(shape);
  return launch_scan_v2(
      scan_args(d, xbc, dt_raw, T, dt_bias, A_q, D_q, exps, X, state, y, nullptr, e_tok), B, w,
      (cudaStream_t)stream);
}

// ------------------------------------------------------------------ chunked scan mode
namespace {
struct SsdWs {
  float *dH;
  float *achunk;
  uint16_t *Hin;
};
SsdWs carve_ssd(Carver &c, const Dims &d, int B, int T) {
  const long long nch = (T + kSsdQ - 1) / kSsdQ, units = (long long)B * d.nh * nch;
  SsdWs w;
  w.dH = c.take<float>(units * kSsdHd * kSsdDs);
  w.achunk = c.take<float>(units);
  w.Hin = c.take<uint16_t>(units * kSsdHd * kSsdDs);
  return w;
}
}  // namespace

extern "C" size_t fm_ssd_workspace_bytes(const fm_shape *shape, int B, int T) {
  Dims d;
  if (check_shape(shape, &d, __func__) != FM_OK || B < 0 || T < 0) return 0;
  Carver c{nullptr, 0};
  carve_ssd(c, d, B, T);
  return c.off + 256;
}

static fm_status launch_ssd(const Dims &d, const int8_t *xbc, const float *dt_raw, int B, int T,
                            const float *dt_bias, const int32_t *A_q, const int32_t *D_q,
                            const int32_t *exps, const fm_exp_layout &X, int32_t *state,
                            int32_t *y, const SsdWs &w, cudaStream_t s);

extern "C" fm_status fm_ssd_scan(const int8_t *xbc, const float *dt_raw, int B, int T,
                                 const fm_shape *shape, const float *dt_bias, const int32_t *A_q,
                                 const int32_t *D_q, const int32_t *exps, int32_t *state,
                                 int32_t *y, void *ws, size_t ws_bytes, fm_stream stream) {
  Dims d;
  FM_TRY(check_shape(shape, &d, __func__));
  if (B < 0 || T < 0) return fail(FM_ERR_SHAPE, "fm_ssd_scan: B, T must be >= 0");
  if ((long long)B * T == 0) return FM_OK;
  if (B > 65535) return fail(FM_ERR_SHAPE, "fm_ssd_scan: B=%d exceeds 65535", B);
  NEED(xbc);
  NEED(dt_raw);
  NEED(dt_bias);
  NEED(A_q);
  NEED(D_q);
  NEED(exps);
  NEED(y);
  OPT(state);
  if (d.cc % 16) return fail(FM_ERR_ALIGNMENT, "fm_ssd_scan: conv channels must be a multiple of 16");
  if (state16())
    return fail(FM_ERR_UNSUPPORTED, "fm_ssd_scan: the chunked scan carries the int32 state word; "
                "the 16-bit state spec is not supported in this mode");
  const size_t need = fm_ssd_workspace_bytes(shape, B, T);
  if (!ws || ws_bytes < need || !aligned16(ws))
    return fail(FM_ERR_WORKSPACE, "fm_ssd_scan: workspace needs %zu bytes", need);
  Carver c{reinterpret_cast<uint8_t *>(ws), 0};
  const SsdWs w = carve_ssd(c, d, B, T);
  return launch_ssd(d, xbc, dt_raw, B, T, dt_bias, A_q, D_q, exps, fm_exp_table_layout(shape),
                    state, y, w, (cudaStream_t)stream);
}

static fm_status launch_ssd(const Dims &d, const int8_t *xbc, const float *dt_raw, int B, int T,
                            const float *dt_bias, const int32_t *A_q, const int32_t *D_q,
                            const int32_t *exps, const fm_exp_layout &X, int32_t *state,
                            int32_t *y, const SsdWs &w, cudaStream_t s) {
  SsdArgs a;
  a.xbc = xbc;
  a.dt_raw = dt_raw;
  a.T = T;
  a.nh = d.nh;
  a.cc = d.cc;
  a.di = d.di;
  a.nch = (T + kSsdQ - 1) / kSsdQ;
  a.dt_bias = dt_bias;
  a.A_q = A_q;
  a.D_q = D_q;
  a.e_x = exps + X.e_x;
  a.e_B = exps + X.e_B;
  a.e_C = exps + X.e_C;
  a.e_h = exps + X.e_h;
  a.e_y = exps + X.e_y;
  a.e_D = exps + X.e_D;
  a.state = state;
  a.y = y;
  a.dH = w.dH;
  a.achunk = w.achunk;
  a.Hin = w.Hin;
  const dim3 grid((unsigned)a.nch, (unsigned)d.nh, (unsigned)B);
  FM_CHECK_CUDA(cudaFuncSetAttribute(k_ssd_state, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     SsdStateSmem::kBytes));
  FM_CHECK_CUDA(cudaFuncSetAttribute(k_ssd_out, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     SsdOutSmem::kBytes));
  FM_TRY(launch_ex("k_ssd_state", k_ssd_state, grid, kSsdThreads, SsdStateSmem::kBytes, s, a));
  FM_TRY(launched("k_ssd_state"));
  FM_TRY(launch_ex("k_ssd_pass", k_ssd_pass,
                   dim3(kSsdHd * kSsdDs / 256, (unsigned)d.nh, (unsigned)B), 256, 0, s, a));
  FM_TRY(launched("k_ssd_pass"));
  FM_TRY(launch_ex("k_ssd_out", k_ssd_out, grid, kSsdOutThreads, SsdOutSmem::kBytes, s, a));
  return launched("k_ssd_out");
}

static fm_status gate_impl(const int32_t *y, const float *z, long long M, const Dims &d,
                           const int32_t *exps, const fm_exp_layout &X, const float *norm_w,
                           int rotate, int mode, const float *static_amax, int8_t *q, float *s_x,
                           float *amax_row, unsigned long long *gstat, const int32_t *e_g_override,
                           cudaStream_t s) {
  if (M <= 0) return FM_OK;
  const int nb = d.di / 256;
  if (nb % 2 == 0 && M >= 2LL * sm_count())
    FM_TRY(launch_ex("k_gate_norm_quant", k_gate_norm_quant<2>, (unsigned)M, 32 * (nb / 2), 0, s, y,
                     z, d.di, d.hd, exps + X.e_y, e_g_override ? e_g_override : exps + X.e_g,
                     norm_w, rotate, mode, static_amax, q, s_x, amax_row, gstat));
  else
    FM_TRY(launch_ex("k_gate_norm_quant", k_gate_norm_quant<1>, (unsigned)M, 32 * nb, 0, s, y, z,
                     d.di, d.hd, exps + X.e_y, e_g_override ? e_g_override : exps + X.e_g, norm_w,
                     rotate, mode, static_amax, q, s_x, amax_row, gstat));
  return launched("k_gate_norm_quant");
}

extern "C" fm_status fm_gate_norm_quant(const int32_t *y, const float *z, int64_t M,
                                        const fm_shape *shape, const int32_t *exps,
                                        const float *norm_w, int rotate, int mode,
                                        const float *static_amax, int8_t *q, float *s_x,
                                        float *amax_row, fm_stream stream) {
  Dims d;
  FM_TRY(check_shape(shape, &d, __func__));
  if (M < 0 || M > 2147483647LL) return fail(FM_ERR_SHAPE, "fm_gate_norm_quant: bad M");
  if (mode != FM_DYNAMIC && mode != FM_STATIC)
    return fail(FM_ERR_INVALID_ARG, "fm_gate_norm_quant: bad mode %d", mode);
  if (M == 0) return FM_OK;
  NEED(y);
  NEED(z);
  NEED(exps);
  NEED(norm_w);
  NEED(q);
  NEED(s_x);
  OPT(amax_row);
  if (mode == FM_STATIC && !static_amax)
    return fail(FM_ERR_INVALID_ARG, "fm_gate_norm_quant: static mode needs static_amax");
  return gate_impl(y, z, M, d, exps, fm_exp_table_layout(shape), norm_w, rotate ? 1 : 0, mode,
                   static_amax, q, s_x, amax_row, nullptr, nullptr, (cudaStream_t)stream);
}

__global__ void k_eval_pwl(int kind, const int64_t *in, long long n, int64_t *out) {
  __shared__ int2 tab[8];
  pwl_table_init(tab);
  __syncthreads();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const long long v = in[i];
  long long r = 0;
  switch (kind) {
    case 0: r = pow2_pwl(v); break;
    case 1: r = exp_pwl(v); break;
    case 2: r = softplus_pwl((int)satb64(v, 32)); break;
    case 3: r = silu_pwl_t((int)satb64(v, 32), tab); break;
    default: r = to_q16(__uint_as_float((unsigned int)(v & 0xFFFFFFFFLL))); break;
  }
  out[i] = r;
}

extern "C" fm_status fm_eval_pwl(int kind, const int64_t *in, int64_t n, int64_t *out,
                                 fm_stream stream) {
  if (kind < 0 || kind > 4) return fail(FM_ERR_INVALID_ARG, "fm_eval_pwl: bad kind %d", kind);
  if (n < 0) return fail(FM_ERR_SHAPE, "fm_eval_pwl: n < 0");
  if (n == 0) return FM_OK;
  NEED(in);
  NEED(out);
  k_eval_pwl<<<(unsigned)((n + 255) / 256), 256, 0, (cudaStream_t)stream>>>(kind, in, n, out);
  return launched("k_eval_pwl");
}

// ------------------------------------------------------------------ layers
namespace {
struct MixerWs {
  int8_t *q_in;
  float *sx_in;
  float *z;
  int8_t *xbc;
  float *dt;
  int8_t *xo;
  int32_t *y;
  int8_t *q_out;
  float *sx_out;
  ScanWs scan;
  int32_t *e_tok;  // [M, nh + 2] per-token conv-output exponents (per-token mode only)
  SsdWs ssd;  // chunked scan mode only (null otherwise)
  int32_t *split;  // split-K partial sums of the small-grid GEMMs (null when none split)
};

MixerWs carve_mixer(Carver &c, const Dims &d, int B, int T) {
  const long long M = (long long)B * T;
  MixerWs w;
  w.q_in = c.take<int8_t>(M * d.dm);
  w.sx_in = c.take<float>(M);
  w.z = c.take<float>(M * d.di);
  w.xbc = c.take<int8_t>(M * d.cc);
  w.dt = c.take<float>(M * d.nh);
  w.xo = c.take<int8_t>(M * d.cc);
  w.y = c.take<int32_t>(M * d.di);
  w.q_out = c.take<int8_t>(M * d.di);
  w.sx_out = c.take<float>(M);
  w.scan = carve_scan(c, d, B, T, xbc_tok());
  w.e_tok = xbc_tok() ? c.take<int32_t>(M * (d.nh + 2)) : nullptr;
  if (use_ssd(T)) {
    w.ssd = carve_ssd(c, d, B, T);
  } else {
    w.ssd.dH = w.ssd.achunk = nullptr;
    w.ssd.Hin = nullptr;
  }
  const bool in_split = gemm_would_split(M, d.n_in, d.dm);
  const bool out_split = gemm_would_split(M, d.dm, d.di);
  const long long n = in_split ? (out_split ? (d.n_in > d.dm ? d.n_in : d.dm) : d.n_in)
                               : (out_split ? d.dm : 0);
  w.split = n ? c.take<int32_t>(M * n) : nullptr;
  return w;
}
}  // namespace

extern "C" size_t fm_workspace_bytes(const fm_shape *shape, int B, int T) {
  Dims d;
  if (check_shape(shape, &d, __func__) != FM_OK || B < 0 || T < 0) return 0;
  Carver c{nullptr, 0};
  carve_mixer(c, d, B, T);
  return c.off + 256;
}

static fm_status check_layer(const fm_layer *L, Dims *d, const char *fn) {
  if (!L) return fail(FM_ERR_INVALID_ARG, "%s: layer is null", fn);
  FM_TRY(check_shape(&L->shape, d, fn));
  if (L->mode != FM_DYNAMIC && L->mode != FM_STATIC)
    return fail(FM_ERR_INVALID_ARG, "%s: bad mode %d", fn, L->mode);
  const void *req[] = {L->w_in_q, L->w_in_s, L->w_out_q, L->w_out_s, L->conv_wq, L->conv_bq,
                       L->dt_bias, L->A_q, L->D_q, L->norm_w, L->exps};
  for (const void *p : req) {
    if (!p) return fail(FM_ERR_INVALID_ARG, "%s: a required layer pointer is null", fn);
    if (!aligned16(p)) return fail(FM_ERR_ALIGNMENT, "%s: a layer pointer is misaligned", fn);
  }
  if (L->mode == FM_STATIC && !L->static_amax)
    return fail(FM_ERR_INVALID_ARG, "%s: static mode needs static_amax", fn);
  if (L->prenorm_w && !aligned16(L->prenorm_w))
    return fail(FM_ERR_ALIGNMENT, "%s: prenorm_w misaligned", fn);
  return FM_OK;
}

// Launch limits of the whole layer, checked before its first kernel: B is a
// grid dimension of the conv and the scan (<= 65535); B * T rows feed the
// GEMMs, whose row-tile count is bounded by 65535.
static fm_status check_batch(int B, int T, const char *fn) {
  if (B > 65535) return fail(FM_ERR_SHAPE, "%s: B=%d exceeds 65535", fn, B);
  if ((long long)B * T > 65535LL * kGemmBM)
    return fail(FM_ERR_SHAPE, "%s: B*T=%lld exceeds %lld rows", fn, (long long)B * T,
                65535LL * kGemmBM);
  return FM_OK;
}

// Hand-over points of one run of a pipelined stack prefill (fm_stack_prefill):
// before its conv the stream waits for the previous run's conv of the layer
// (which wrote the conv state this run reads), after it records its own; the
// same around the scan for the SSM state.  A null event is skipped.
struct StageSync {
  cudaEvent_t conv_wait, conv_done, scan_wait, scan_done;
};

static fm_status sync_wait(const StageSync *sy, cudaEvent_t StageSync::*ev, cudaStream_t s) {
  if (sy && sy->*ev) {
    FM_CHECK_CUDA(cudaStreamWaitEvent(s, sy->*ev, 0));
    t_after_cross_wait = true;
  }
  return FM_OK;
}
static fm_status sync_record(const StageSync *sy, cudaEvent_t StageSync::*ev, cudaStream_t s) {
  if (sy && sy->*ev) FM_CHECK_CUDA(cudaEventRecord(sy->*ev, s));
  return FM_OK;
}

static fm_status mixer_impl(const fm_layer *L, const Dims &d, const float *x, int B, int T,
                            int residual, int8_t *conv_state, int32_t *ssm_state, float *out,
                            const MixerWs &w, cudaStream_t s, const StageSync *sync = nullptr) {
  const long long M = (long long)B * T;
  const fm_exp_layout X = fm_exp_table_layout(&L->shape);
  const float *amax_in = L->static_amax, *amax_out = L->static_amax ? L->static_amax + 1 : nullptr;
  FM_TRY(launch_hadamard_quant(x, M, d.dm, L->prenorm_w, L->rotate, L->mode, amax_in, w.q_in,
                               w.sx_in, nullptr, s));
  FM_TRY(in_proj_impl(w.q_in, w.sx_in, M, L->w_in_q, L->w_in_s, d, L->exps + X.e_u, w.z, w.xbc,
                      w.dt, s, w.split));
  FM_TRY(sync_wait(sync, &StageSync::conv_wait, s));
  FM_TRY(launch_conv(w.xbc, B, T, d.cc, L->conv_wq, L->conv_bq, L->exps, conv_state, w.xo,
                     nullptr, s, w.e_tok, &d));
  FM_TRY(sync_record(sync, &StageSync::conv_done, s));
  if (w.ssd.dH && (state16() || w.e_tok))
    return fail(FM_ERR_UNSUPPORTED, "the chunked scan mode carries the int32 state at static "
                "exponents: the 16-bit state spec and per-token exponents are not supported");
  FM_TRY(sync_wait(sync, &StageSync::scan_wait, s));
  if (w.ssd.dH)
    FM_TRY(launch_ssd(d, w.xo, w.dt, B, T, L->dt_bias, L->A_q, L->D_q, L->exps, X, ssm_state, w.y,
                      w.ssd, s));
  else
    FM_TRY(launch_scan_v2(scan_args(d, w.xo, w.dt, T, L->dt_bias, L->A_q, L->D_q, L->exps, X,
                                    ssm_state, w.y, nullptr, w.e_tok),
                          B, w.scan, s));
  FM_TRY(sync_record(sync, &StageSync::scan_done, s));
  FM_TRY(gate_impl(w.y, w.z, M, d, L->exps, X, L->norm_w, L->rotate, L->mode, amax_out, w.q_out,
                   w.sx_out, nullptr, nullptr, nullptr, s));
  return launch_gemm(w.q_out, M, L->w_out_q, d.dm, d.di,
                     plain_epilogue(M, d.dm, w.sx_out, L->w_out_s, residual ? x : nullptr, out,
                                    nullptr),
                     s, w.split);
}

extern "C" fm_status fm_mixer_prefill(const fm_layer *L, const float *x, int B, int T,
                                      int residual, int8_t *conv_state, int32_t *ssm_state,
                                      float *out, void *ws, size_t ws_bytes, fm_stream stream) {
  Dims d;
  FM_TRY(check_layer(L, &d, __func__));
  if (B < 0 || T < 0) return fail(FM_ERR_SHAPE, "fm_mixer_prefill: B, T must be >= 0");
  if ((long long)B * T == 0) return FM_OK;
  FM_TRY(check_batch(B, T, __func__));
  NEED(x);
  NEED(out);
  OPT(conv_state);
  OPT(ssm_state);
  const size_t need = fm_workspace_bytes(&L->shape, B, T);
  if (!ws || ws_bytes < need)
    return fail(FM_ERR_WORKSPACE, "fm_mixer_prefill: workspace needs %zu bytes", need);
  if (out != x) {
    const char *xb = reinterpret_cast<const char *>(x), *ob = reinterpret_cast<const char *>(out);
    const size_t bytes = (size_t)B * T * d.dm * sizeof(float);
    if (ob < xb + bytes && xb < ob + bytes)
      return fail(FM_ERR_INVALID_ARG, "fm_mixer_prefill: out partially overlaps x");
  }
  Carver c{reinterpret_cast<uint8_t *>(ws), 0};
  if (!aligned16(ws)) return fail(FM_ERR_ALIGNMENT, "fm_mixer_prefill: ws misaligned");
  const MixerWs w = carve_mixer(c, d, B, T);
  return mixer_impl(L, d, x, B, T, residual, conv_state, ssm_state, out, w, (cudaStream_t)stream);
}

extern "C" fm_status fm_decode_step(const fm_layer *L, const float *x, int B, int residual,
                                    int8_t *conv_state, int32_t *ssm_state, float *out, void *ws,
                                    size_t ws_bytes, fm_stream stream) {
  if (!conv_state || !ssm_state)
    return fail(FM_ERR_INVALID_ARG, "fm_decode_step: conv_state and ssm_state are required");
  return fm_mixer_prefill(L, x, B, 1, residual, conv_state, ssm_state, out, ws, ws_bytes, stream);
}

// ------------------------------------------------------------------ allocation-free decode
// Scratch for fm_decode_step_noalloc: a fixed device array instead of a
// caller workspace, for callers that cannot allocate device memory.  Host
// code only sees a stand-in for this symbol; its device address comes from
// cudaGetSymbolAddress, with the device current.
static __device__ __align__(256) uint8_t g_noalloc_scratch[FM_NOALLOC_SCRATCH_BYTES];

// The address is looked up once per CUDA context and cached under the
// context's unique id (cuCtxGetId).  A context torn down and created again
// (cudaDeviceReset, then the next call) has a new id, so the module's new
// address is looked up again instead of reusing a stale one.  Without the
// driver's context ids the address is looked up on every call.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

static bool current_context_id(unsigned long long *id) {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

static fm_status noalloc_scratch_ptr(void **out) {
  constexpr int kSlots = 64;
  static unsigned long long ids[kSlots] = {0};
  static void *addrs[kSlots] = {nullptr};
  static int next = 0;
  static std::mutex mu;
  int devid = 0;
  FM_CHECK_CUDA(cudaGetDevice(&devid));
  // no current context yet (nothing has touched the device): no id, so the
  // lookup below runs, and it makes the primary context current
  unsigned long long id = 0;
  const bool have_id = current_context_id(&id) && id != 0;
  std::lock_guard<std::mutex> lock(mu);
  if (have_id)
    for (int i = 0; i < kSlots; ++i)
      if (ids[i] == id && addrs[i]) {
        *out = addrs[i];
        return FM_OK;
      }
  void *p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || !p)
    return fail(FM_ERR_CUDA, "fm_decode_step_noalloc: cudaGetSymbolAddress on device %d: %s",
                devid, cudaGetErrorString(e));
  if (have_id) {
    ids[next] = id;
    addrs[next] = p;
    next = (next + 1) % kSlots;
  }
  *out = p;
  return FM_OK;
}

extern "C" fm_status fm_decode_step_noalloc(const fm_layer *L, const float *x, int B,
                                            int residual, int8_t *conv_state, int32_t *ssm_state,
                                            float *out, fm_stream stream) {
  Dims d;
  FM_TRY(check_layer(L, &d, __func__));
  if (!conv_state || !ssm_state)
    return fail(FM_ERR_INVALID_ARG, "fm_decode_step_noalloc: conv_state and ssm_state are required");
  if (B < 0) return fail(FM_ERR_SHAPE, "fm_decode_step_noalloc: B must be >= 0");
  if (B == 0) return FM_OK;
  const size_t need = fm_workspace_bytes(&L->shape, B, 1);
  if (need > (size_t)FM_NOALLOC_SCRATCH_BYTES)
    return fail(FM_ERR_WORKSPACE,
                "fm_decode_step_noalloc: batch %d needs %zu bytes of scratch, more than the "
                "fixed %u-byte array (FM_NOALLOC_SCRATCH_BYTES); use fm_decode_step",
                B, need, (unsigned)FM_NOALLOC_SCRATCH_BYTES);
  void *ws = nullptr;
  FM_TRY(noalloc_scratch_ptr(&ws));
  return fm_decode_step(L, x, B, residual, conv_state, ssm_state, out, ws, need, stream);
}

// ------------------------------------------------------------------ stack prefill
// A residual stack over one batch, x <- x + mixer_l(RMSNorm_l(x)) layer by
// layer, optionally pipelined over time.  The recurrence and the conv carry
// state only forward in time, and every other stage is per token, so a
// sequence cut into runs of consecutive tokens gives the same bits when run k
// of a layer starts from the conv and SSM states run k - 1 of that layer left.
// Pipelined, each run walks the layers on one of the library's own streams and
// waits only at those two hand-overs (StageSync), so the scans of successive
// runs overlap each other and the GEMM and row stages of the neighbouring
// runs: at B = 1 the sequential scan alone cannot fill every SM sub-partition
// evenly.
namespace {
constexpr int kStackStreams = 8;     // internal streams per context
constexpr int kStackMaxChunks = 64;  // runs per sequence

struct StackPlan {
  int runs;     // runs per sequence
  int tc;       // tokens per run (the last run of a sequence may be shorter)
  int chains;   // B * runs, issued in this order: run k of sequence b is b * runs + k
  int streams;  // internal streams in use
};

// runs of ceil(T / n_chunks) tokens rounded up to the scan's 32-token tile
StackPlan stack_plan(int B, int T, int n_chunks) {
  StackPlan p;
  long long tc = ((long long)T + n_chunks - 1) / n_chunks;
  tc = (tc + kPrepTT - 1) / kPrepTT * kPrepTT;
  if (tc > T) tc = T;
  p.tc = (int)tc;
  p.runs = (int)(((long long)T + tc - 1) / tc);
  p.chains = B * p.runs;
  p.streams = p.chains < kStackStreams ? p.chains : kStackStreams;
  return p;
}

size_t ssm_state_bytes_per_seq(const Dims &d) {
  return (size_t)d.nh * d.hd * d.ds * (state16() ? sizeof(int16_t) : sizeof(int32_t));
}

// Pipelined workspace: one mixer workspace (for one run) per internal stream,
// then zero-started conv and SSM states for every layer and sequence, used
// when the caller passes none.
struct StackWs {
  uint8_t *run_ws[kStackStreams];
  size_t run_bytes;
  int8_t *conv;
  uint8_t *ssm;
  size_t conv_bytes, ssm_bytes;
};

StackWs carve_stack(Carver &c, const fm_shape *shape, const Dims &d, int n_layers, int B,
                    const StackPlan &p) {
  StackWs w;
  w.run_bytes = fm_workspace_bytes(shape, 1, p.tc);
  for (int i = 0; i < kStackStreams; ++i)
    w.run_ws[i] = i < p.streams ? c.take<uint8_t>(w.run_bytes) : nullptr;
  w.conv_bytes = (size_t)n_layers * B * 3 * d.cc;
  w.ssm_bytes = (size_t)n_layers * B * ssm_state_bytes_per_seq(d);
  w.conv = c.take<int8_t>(w.conv_bytes);
  w.ssm = c.take<uint8_t>(w.ssm_bytes);
  return w;
}

// The internal streams and events of one CUDA context, created on first use
// and kept for the process (keyed by the context's unique id, so a context
// created anew gets new ones).  The mutex makes each call's host-side issue
// atomic: the events are reused from call to call.
struct StackPool {
  unsigned long long ctx = 0;
  int dev = -1;
  cudaStream_t s[kStackStreams];
  cudaEvent_t fork, joined[kStackStreams], conv_ev[2], scan_ev[2];
  std::mutex mu;
};

fm_status stack_pool(StackPool **out) {
  static std::mutex mu;
  static std::vector<std::unique_ptr<StackPool>> pools;
  int dev = 0;
  FM_CHECK_CUDA(cudaGetDevice(&dev));
  unsigned long long id = 0;
  const bool have_id = current_context_id(&id) && id != 0;
  std::lock_guard<std::mutex> lock(mu);
  for (auto &p : pools)
    if (have_id ? p->ctx == id : p->dev == dev) {
      *out = p.get();
      return FM_OK;
    }
  std::unique_ptr<StackPool> p(new StackPool);
  p->ctx = have_id ? id : 0;
  p->dev = dev;
  for (int i = 0; i < kStackStreams; ++i) {
    FM_CHECK_CUDA(cudaStreamCreateWithFlags(&p->s[i], cudaStreamNonBlocking));
    FM_CHECK_CUDA(cudaEventCreateWithFlags(&p->joined[i], cudaEventDisableTiming));
  }
  FM_CHECK_CUDA(cudaEventCreateWithFlags(&p->fork, cudaEventDisableTiming));
  for (int i = 0; i < 2; ++i) {
    FM_CHECK_CUDA(cudaEventCreateWithFlags(&p->conv_ev[i], cudaEventDisableTiming));
    FM_CHECK_CUDA(cudaEventCreateWithFlags(&p->scan_ev[i], cudaEventDisableTiming));
  }
  *out = p.get();
  pools.push_back(std::move(p));
  return FM_OK;
}
}  // namespace

extern "C" size_t fm_stack_workspace_bytes(const fm_shape *shape, int n_layers, int B, int T,
                                           int n_chunks) {
  Dims d;
  if (check_shape(shape, &d, __func__) != FM_OK || n_layers < 0 || B < 0 || T < 0 ||
      n_chunks < 1 || n_chunks > kStackMaxChunks)
    return 0;
  if (n_chunks == 1 || (long long)B * T == 0) return fm_workspace_bytes(shape, B, T);
  Carver c{nullptr, 0};
  carve_stack(c, shape, d, n_layers, B, stack_plan(B, T, n_chunks));
  return c.off + 256;
}

// The pipelined issue: layer by layer, and within a layer run by run, so that
// each hand-over event is waited on before the next run of the same kind
// records it again (two events of each kind alternate between neighbouring
// runs).  Runs of different sequences share nothing and do not wait.
static fm_status stack_issue(const fm_layer *const *layers, int n_layers, const Dims &d, float *x,
                             const float *x_host, float *out_host, int B, int T,
                             int8_t *const *conv_states, int32_t *const *ssm_states,
                             const StackPlan &p, const StackWs &w, StackPool &pool) {
  struct RunFlag {  // the scan tile rule of pipelined runs, for this call only
    RunFlag() { t_pipelined_run = true; }
    ~RunFlag() { t_pipelined_run = false; }
  } run_flag;
  const size_t conv_seq = (size_t)3 * d.cc, ssm_seq = ssm_state_bytes_per_seq(d);
  for (int l = 0; l < n_layers; ++l)
    for (int c = 0; c < p.chains; ++c) {
      const int b = c / p.runs, k = c % p.runs;
      const int t0 = k * p.tc, tn = (T - t0) < p.tc ? (T - t0) : p.tc;
      cudaStream_t rs = pool.s[c % p.streams];
      float *xr = x + ((long long)b * T + t0) * d.dm;
      int8_t *cs = (conv_states ? conv_states[l] : w.conv + (size_t)l * B * conv_seq) + b * conv_seq;
      uint8_t *sb = ssm_states ? reinterpret_cast<uint8_t *>(ssm_states[l])
                               : w.ssm + (size_t)l * B * ssm_seq;
      int32_t *ss = reinterpret_cast<int32_t *>(sb + (size_t)b * ssm_seq);
      StageSync sy;
      sy.conv_wait = k > 0 ? pool.conv_ev[(c - 1) & 1] : nullptr;
      sy.scan_wait = k > 0 ? pool.scan_ev[(c - 1) & 1] : nullptr;
      sy.conv_done = k + 1 < p.runs ? pool.conv_ev[c & 1] : nullptr;
      sy.scan_done = k + 1 < p.runs ? pool.scan_ev[c & 1] : nullptr;
      Carver rc{w.run_ws[c % p.streams], 0};
      const MixerWs mw = carve_mixer(rc, d, 1, tn);
      const size_t run_bytes = (size_t)tn * d.dm * sizeof(float);
      const long long row0 = (long long)b * T + t0;
      if (l == 0 && x_host)  // this run's input, on its own stream
        FM_CHECK_CUDA(cudaMemcpyAsync(xr, x_host + row0 * d.dm, run_bytes, cudaMemcpyHostToDevice,
                                      rs));
      FM_TRY(mixer_impl(layers[l], d, xr, 1, tn, 1, cs, ss, xr, mw, rs, &sy));
      if (l == n_layers - 1 && out_host)  // and its output, as soon as it is final
        FM_CHECK_CUDA(cudaMemcpyAsync(out_host + row0 * d.dm, xr, run_bytes,
                                      cudaMemcpyDeviceToHost, rs));
    }
  return FM_OK;
}

// The stack on device rows x; with x_host / out_host (host) the input is
// copied in and the output out inside the same schedule (per run when
// pipelined, so the copies of one run overlap the other runs' kernels).
static fm_status stack_prefill(const char *fn, const fm_layer *const *layers, int n_layers,
                               float *x, const float *x_host, float *out_host, int B, int T,
                               int8_t *const *conv_states, int32_t *const *ssm_states,
                               int n_chunks, void *ws, size_t ws_bytes, cudaStream_t s) {
  if (n_layers < 0) return fail(FM_ERR_INVALID_ARG, "%s: n_layers < 0", fn);
  if (n_chunks < 1 || n_chunks > kStackMaxChunks)
    return fail(FM_ERR_INVALID_ARG, "%s: n_chunks=%d is not in [1, %d]", fn, n_chunks,
                kStackMaxChunks);
  if (B < 0 || T < 0) return fail(FM_ERR_SHAPE, "%s: B, T must be >= 0", fn);
  if ((long long)B * T == 0) return FM_OK;
  if (!x) return fail(FM_ERR_INVALID_ARG, "%s: the device rows x are null", fn);
  if (!aligned16(x)) return fail(FM_ERR_ALIGNMENT, "%s: x is not 16-byte aligned", fn);
  if (n_layers == 0) return FM_OK;  // no layer: nothing to do (no width to copy either)
  if (!layers) return fail(FM_ERR_INVALID_ARG, "%s: layers is null", fn);
  Dims d;
  FM_TRY(check_layer(layers[0], &d, fn));
  for (int l = 0; l < n_layers; ++l) {
    Dims dl;
    FM_TRY(check_layer(layers[l], &dl, fn));
    const fm_shape &a = layers[0]->shape, &sh = layers[l]->shape;
    if (a.d_model != sh.d_model || a.d_inner != sh.d_inner)
      return fail(FM_ERR_SHAPE, "%s: layer %d's shape differs from layer 0's", fn, l);
    if (conv_states && (!conv_states[l] || !aligned16(conv_states[l])))
      return fail(FM_ERR_INVALID_ARG, "%s: conv_states[%d] is null or misaligned", fn, l);
    if (ssm_states && (!ssm_states[l] || !aligned16(ssm_states[l])))
      return fail(FM_ERR_INVALID_ARG, "%s: ssm_states[%d] is null or misaligned", fn, l);
  }
  FM_TRY(check_batch(B, T, fn));
  const size_t need = fm_stack_workspace_bytes(&layers[0]->shape, n_layers, B, T, n_chunks);
  if (!ws || ws_bytes < need)
    return fail(FM_ERR_WORKSPACE, "%s: workspace needs %zu bytes", fn, need);
  if (!aligned16(ws)) return fail(FM_ERR_ALIGNMENT, "%s: ws misaligned", fn);
  const size_t all_bytes = (size_t)B * T * d.dm * sizeof(float);
  Carver c{reinterpret_cast<uint8_t *>(ws), 0};
  if (n_chunks == 1) {  // the plain layer loop on the caller's stream
    if (x_host) FM_CHECK_CUDA(cudaMemcpyAsync(x, x_host, all_bytes, cudaMemcpyHostToDevice, s));
    const MixerWs w = carve_mixer(c, d, B, T);
    for (int l = 0; l < n_layers; ++l)
      FM_TRY(mixer_impl(layers[l], d, x, B, T, 1, conv_states ? conv_states[l] : nullptr,
                        ssm_states ? ssm_states[l] : nullptr, x, w, s));
    if (out_host) FM_CHECK_CUDA(cudaMemcpyAsync(out_host, x, all_bytes, cudaMemcpyDeviceToHost, s));
    return FM_OK;
  }
  const StackPlan p = stack_plan(B, T, n_chunks);
  const StackWs w = carve_stack(c, &layers[0]->shape, d, n_layers, B, p);
  if (!conv_states) FM_CHECK_CUDA(cudaMemsetAsync(w.conv, 0, w.conv_bytes, s));
  if (!ssm_states) FM_CHECK_CUDA(cudaMemsetAsync(w.ssm, 0, w.ssm_bytes, s));
  StackPool *pool = nullptr;
  FM_TRY(stack_pool(&pool));
  std::lock_guard<std::mutex> lock(pool->mu);
  FM_CHECK_CUDA(cudaEventRecord(pool->fork, s));
  for (int i = 0; i < p.streams; ++i) FM_CHECK_CUDA(cudaStreamWaitEvent(pool->s[i], pool->fork, 0));
  const fm_status st = stack_issue(layers, n_layers, d, x, x_host, out_host, B, T, conv_states,
                                   ssm_states, p, w, *pool);
  // joined back even after a failed launch, so that the caller's stream never
  // runs ahead of work already queued on the internal streams
  for (int i = 0; i < p.streams; ++i) {
    FM_CHECK_CUDA(cudaEventRecord(pool->joined[i], pool->s[i]));
    FM_CHECK_CUDA(cudaStreamWaitEvent(s, pool->joined[i], 0));
  }
  return st;
}

extern "C" fm_status fm_stack_prefill(const fm_layer *const *layers, int n_layers, float *x,
                                      int B, int T, int8_t *const *conv_states,
                                      int32_t *const *ssm_states, int n_chunks, void *ws,
                                      size_t ws_bytes, fm_stream stream) {
  return stack_prefill(__func__, layers, n_layers, x, nullptr, nullptr, B, T, conv_states,
                       ssm_states, n_chunks, ws, ws_bytes, (cudaStream_t)stream);
}

extern "C" fm_status fm_stack_prefill_host(const fm_layer *const *layers, int n_layers,
                                           const float *x_host, float *out_host, float *x_dev,
                                           int B, int T, int8_t *const *conv_states,
                                           int32_t *const *ssm_states, int n_chunks, void *ws,
                                           size_t ws_bytes, fm_stream stream) {
  if ((long long)B * T > 0 && (!x_host || !out_host))
    return fail(FM_ERR_INVALID_ARG, "fm_stack_prefill_host: x_host and out_host are required");
  return stack_prefill(__func__, layers, n_layers, x_dev, x_host, out_host, B, T, conv_states,
                       ssm_states, n_chunks, ws, ws_bytes, (cudaStream_t)stream);
}

// ------------------------------------------------------------------ FastMamba-LQ
static fm_status lq_check_params(const fm_lq_params *P, const char *fn) {
  if (!P) return fail(FM_ERR_INVALID_ARG, "%s: params is null", fn);
  const void *req[] = {P->conv_w, P->conv_b, P->a_log, P->D};
  for (const void *p : req) {
    if (!p) return fail(FM_ERR_INVALID_ARG, "%s: a required LQ parameter pointer is null", fn);
    if (!aligned16(p)) return fail(FM_ERR_ALIGNMENT, "%s: an LQ parameter pointer is misaligned", fn);
  }
  return FM_OK;
}

static fm_status launch_lq_conv(const float *u, long long ldu, int B, int T, int cc,
                                const float *w, const float *bias, float *conv_state, float *out,
                                cudaStream_t s) {
  const dim3 grid((unsigned)((T + kLqConvTT - 1) / kLqConvTT), (unsigned)((cc + 255) / 256),
                  (unsigned)B);
  FM_TRY(launch_ex("k_lq_conv", k_lq_conv, grid, 256, 0, s, u, ldu, T, cc, w, bias, conv_state,
                   out));
  FM_TRY(launched("k_lq_conv"));
  if (conv_state) {
    const long long n = (long long)B * cc;
    FM_TRY(launch_ex("k_lq_conv_state_update", k_lq_conv_state_update, (unsigned)((n + 255) / 256),
                     256, 0, s, u, ldu, B, T, cc, conv_state));
    FM_TRY(launched("k_lq_conv_state_update"));
  }
  return FM_OK;
}

template <int CPW>
static fm_status launch_lq_scan_t(const Dims &d, const float *xo, const float *dt_raw,
                                  long long ld_dt, const float *z, long long ld_z, int B, int T,
                                  const float *dt_bias, const float *a_log, const float *D,
                                  float *state, float *out, cudaStream_t s) {
  constexpr int smem = (int)sizeof(LqScanSmem<CPW>);
  FM_CHECK_CUDA(cudaFuncSetAttribute(k_lq_scan<CPW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     smem));
  FM_TRY(launch_ex("k_lq_scan", k_lq_scan<CPW>,
                   dim3((unsigned)(d.hd / (4 * CPW)), (unsigned)d.nh, (unsigned)B), 128, smem, s,
                   xo, dt_raw, ld_dt, z, ld_z, T, d.nh, d.cc, d.di, dt_bias, a_log, D, state, out));
  return launched("k_lq_scan");
}

// Channels per warp of the LQ scan, process-wide: 0 (default) chooses by the
// grid, 1, 2 or 4 forces it (tuning; the same results either way up to the
// warp reduction's order).
static std::atomic<int> g_lq_cpw{0};

extern "C" fm_status fm_set_lq_scan_cpw(int cpw) {
  if (cpw != 0 && cpw != 1 && cpw != 2 && cpw != 4)
    return fail(FM_ERR_INVALID_ARG, "fm_set_lq_scan_cpw: %d is not 0, 1, 2 or 4", cpw);
  g_lq_cpw.store(cpw, std::memory_order_relaxed);
  return FM_OK;
}

static fm_status launch_lq_scan(const Dims &d, const float *xo, const float *dt_raw,
                                long long ld_dt, const float *z, long long ld_z, int B, int T,
                                const float *dt_bias, const float *a_log, const float *D,
                                float *state, float *out, cudaStream_t s) {
  // Each warp re-reads the staged B and C rows of every step for its CPW
  // channels, so wider warps cut the shared-memory traffic per state cell,
  // but the recurrence's latency wants two CTAs on every SM: by default the
  // widest CPW that still gives each SM two (measured on the 24-layer 130M
  // stack, B = 1, T = 2048: 1 / 2 / 4 channels per warp = 7.64 / 8.12 /
  // 9.42 ms per step; 64-layer 2.7B, B = 2, T = 4096: 4 beats 2 by 8 %).
  int cpw = g_lq_cpw.load(std::memory_order_relaxed);
  if (cpw == 0) {
    const long long ctas4 = (long long)B * d.nh * (d.hd / 16), slots = 2LL * sm_count();
    cpw = ctas4 >= slots ? 4 : (2 * ctas4 >= slots ? 2 : 1);
  }
  if (cpw == 4)
    return launch_lq_scan_t<4>(d, xo, dt_raw, ld_dt, z, ld_z, B, T, dt_bias, a_log, D, state,
                               out, s);
  if (cpw == 2)
    return launch_lq_scan_t<2>(d, xo, dt_raw, ld_dt, z, ld_z, B, T, dt_bias, a_log, D, state,
                               out, s);
  return launch_lq_scan_t<1>(d, xo, dt_raw, ld_dt, z, ld_z, B, T, dt_bias, a_log, D, state, out,
                             s);
}

extern "C" fm_status fm_lq_conv1d(const float *u, int64_t ldu, int B, int T,
                                  const fm_shape *shape, const float *conv_w,
                                  const float *conv_b, float *conv_state, float *out,
                                  fm_stream stream) {
  Dims d;
  FM_TRY(check_shape(shape, &d, __func__));
  if (B < 0 || T < 0) return fail(FM_ERR_SHAPE, "fm_lq_conv1d: B, T must be >= 0");
  if ((long long)B * T == 0) return FM_OK;
  if (B > 65535) return fail(FM_ERR_SHAPE, "fm_lq_conv1d: B=%d exceeds 65535", B);
  if (ldu < d.cc) return fail(FM_ERR_SHAPE, "fm_lq_conv1d: ldu %lld < conv channels %d",
                              (long long)ldu, d.cc);
  if (!u) return fail(FM_ERR_INVALID_ARG, "fm_lq_conv1d: u is null");
  NEED(conv_w);
  NEED(conv_b);
  NEED(out);
  OPT(conv_state);
  return launch_lq_conv(u, ldu, B, T, d.cc, conv_w, conv_b, conv_state, out,
                        (cudaStream_t)stream);
}

extern "C" fm_status fm_lq_scan(const float *xo, const float *dt_raw, int64_t ld_dt,
                                const float *z, int64_t ld_z, int B, int T,
                                const fm_shape *shape, const float *dt_bias, const float *a_log,
                                const float *D, float *state, float *out, fm_stream stream) {
  Dims d;
  FM_TRY(check_shape(shape, &d, __func__));
  if (B < 0 || T < 0) return fail(FM_ERR_SHAPE, "fm_lq_scan: B, T must be >= 0");
  if ((long long)B * T == 0) return FM_OK;
  if (B > 65535) return fail(FM_ERR_SHAPE, "fm_lq_scan: B=%d exceeds 65535", B);
  if (ld_dt < d.nh || (z && ld_z < d.di))
    return fail(FM_ERR_SHAPE, "fm_lq_scan: row strides too small (ld_dt %lld, ld_z %lld)",
                (long long)ld_dt, (long long)ld_z);
  NEED(xo);
  if (!dt_raw) return fail(FM_ERR_INVALID_ARG, "fm_lq_scan: dt_raw is null");
  NEED(dt_bias);
  NEED(a_log);
  NEED(D);
  NEED(out);
  OPT(state);
  return launch_lq_scan(d, xo, dt_raw, ld_dt, z, ld_z, B, T, dt_bias, a_log, D, state, out,
                        (cudaStream_t)stream);
}

namespace {
struct LqWs {
  int8_t *q_in;
  float *sx_in;
  float *Y;  // [M, n_in] in_proj output: z | xBC | dt_raw
  float *xo;
  float *g;
  int8_t *q_out;
  float *sx_out;
  int32_t *split;
};
LqWs carve_lq(Carver &c, const Dims &d, int B, int T) {
  const long long M = (long long)B * T;
  LqWs w;
  w.q_in = c.take<int8_t>(M * d.dm);
  w.sx_in = c.take<float>(M);
  w.Y = c.take<float>(M * d.n_in);
  w.xo = c.take<float>(M * d.cc);
  w.g = c.take<float>(M * d.di);
  w.q_out = c.take<int8_t>(M * d.di);
  w.sx_out = c.take<float>(M);
  const bool in_split = gemm_would_split(M, d.n_in, d.dm);
  const bool out_split = gemm_would_split(M, d.dm, d.di);
  const long long n = in_split ? (out_split ? (d.n_in > d.dm ? d.n_in : d.dm) : d.n_in)
                               : (out_split ? d.dm : 0);
  w.split = n ? c.take<int32_t>(M * n) : nullptr;
  return w;
}
}  // namespace

extern "C" size_t fm_lq_workspace_bytes(const fm_shape *shape, int B, int T) {
  Dims d;
  if (check_shape(shape, &d, __func__) != FM_OK || B < 0 || T < 0) return 0;
  Carver c{nullptr, 0};
  carve_lq(c, d, B, T);
  return c.off + 256;
}

extern "C" fm_status fm_lq_mixer_prefill(const fm_layer *L, const fm_lq_params *P,
                                         const float *x, int B, int T, int residual,
                                         float *conv_state, float *ssm_state, float *out,
                                         void *ws, size_t ws_bytes, fm_stream stream) {
  Dims d;
  FM_TRY(check_layer(L, &d, __func__));
  FM_TRY(lq_check_params(P, __func__));
  if (B < 0 || T < 0) return fail(FM_ERR_SHAPE, "fm_lq_mixer_prefill: B, T must be >= 0");
  if ((long long)B * T == 0) return FM_OK;
  FM_TRY(check_batch(B, T, __func__));
  NEED(x);
  NEED(out);
  OPT(conv_state);
  OPT(ssm_state);
  const size_t need = fm_lq_workspace_bytes(&L->shape, B, T);
  if (!ws || ws_bytes < need || !aligned16(ws))
    return fail(FM_ERR_WORKSPACE, "fm_lq_mixer_prefill: workspace needs %zu bytes", need);
  if (out != x) {
    const char *xb = reinterpret_cast<const char *>(x), *ob = reinterpret_cast<const char *>(out);
    const size_t bytes = (size_t)B * T * d.dm * sizeof(float);
    if (ob < xb + bytes && xb < ob + bytes)
      return fail(FM_ERR_INVALID_ARG, "fm_lq_mixer_prefill: out partially overlaps x");
  }
  Carver c{reinterpret_cast<uint8_t *>(ws), 0};
  const LqWs w = carve_lq(c, d, B, T);
  const cudaStream_t s = (cudaStream_t)stream;
  const long long M = (long long)B * T;
  const float *amax_in = L->static_amax, *amax_out = L->static_amax ? L->static_amax + 1 : nullptr;
  // rotated W8A8 in_proj with a plain fp32 output
  FM_TRY(launch_hadamard_quant(x, M, d.dm, L->prenorm_w, L->rotate, L->mode, amax_in, w.q_in,
                               w.sx_in, nullptr, s));
  FM_TRY(launch_gemm(w.q_in, M, L->w_in_q, d.n_in, d.dm,
                     plain_epilogue(M, d.n_in, w.sx_in, L->w_in_s, nullptr, w.Y, nullptr), s,
                     w.split));
  // exact fp32 conv, scan and gate
  FM_TRY(launch_lq_conv(w.Y + d.di, d.n_in, B, T, d.cc, P->conv_w, P->conv_b, conv_state, w.xo,
                        s));
  FM_TRY(launch_lq_scan(d, w.xo, w.Y + d.di + d.cc, d.n_in, w.Y, d.n_in, B, T, L->dt_bias,
                        P->a_log, P->D, ssm_state, w.g, s));
  // gated RMSNorm (the norm weight as the pre-norm weight), rotation, int8
  FM_TRY(launch_hadamard_quant(w.g, M, d.di, L->norm_w, L->rotate, L->mode, amax_out, w.q_out,
                               w.sx_out, nullptr, s));
  return launch_gemm(w.q_out, M, L->w_out_q, d.dm, d.di,
                     plain_epilogue(M, d.dm, w.sx_out, L->w_out_s, residual ? x : nullptr, out,
                                    nullptr),
                     s, w.split);
}

// ------------------------------------------------------------------ offline preparation
__global__ void k_prepare_mixer_params(const float *conv_w, const float *a_log, const float *D,
                                       int cc, int nh, int8_t *conv_wq, int32_t *A_q,
                                       int32_t *D_q, int32_t *e_w, int32_t *e_D) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < cc) {
    double amax = 0.0;
    for (int k = 0; k < 4; ++k) amax = fmax(amax, fabs((double)conv_w[i * 4 + k]));
    const int e = pot_exponent(amax, 127.0);
    e_w[i] = e;
    for (int k = 0; k < 4; ++k)
      conv_wq[i * 4 + k] = (int8_t)round_clamp(__fmul_rn(conv_w[i * 4 + k], ldexpf(1.0f, -e)), 127.0f);
  }
  if (i < nh) {
    // A_q = rint(exp(A_log) log2(e) 2^12): A = -exp(A_log) folded with log2(e)
    A_q[i] = (int32_t)llrint(__dmul_rn(__ddiv_rn(exp((double)a_log[i]), 0.69314718055994530942), 4096.0));
    const int e = pot_exponent(fabs((double)D[i]), 16384.0);
    e_D[i] = e;
    D_q[i] = (int32_t)satb64(llrint(ldexp((double)D[i], -e)), 16);
  }
}

extern "C" fm_status fm_prepare_mixer_params(const fm_shape *shape, const float *conv_w,
                                             const float *a_log, const float *D, int8_t *conv_wq,
                                             int32_t *A_q, int32_t *D_q, int32_t *exps,
                                             fm_stream stream) {
  Dims d;
  FM_TRY(check_shape(shape, &d, __func__));
  NEED(conv_w);
  NEED(a_log);
  NEED(D);
  NEED(conv_wq);
  NEED(A_q);
  NEED(D_q);
  NEED(exps);
  const fm_exp_layout X = fm_exp_table_layout(shape);
  const int n = d.cc > d.nh ? d.cc : d.nh;
  k_prepare_mixer_params<<<(n + 127) / 128, 128, 0, (cudaStream_t)stream>>>(
      conv_w, a_log, D, d.cc, d.nh, conv_wq, A_q, D_q, exps + X.e_w, exps + X.e_D);
  return launched("k_prepare_mixer_params");
}

// ------------------------------------------------------------------ calibration
// Stage statistics -> exponents, all on the device (see fm_calibrate_layer).
__global__ void k_calib_fill(int32_t *p, int n, int v) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = v;
}
__global__ void k_max_f32(const float *v, long long n, float *out) {
  __shared__ float red[32];
  float m = 0.0f;
  for (long long i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, v[i]);
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = 0.0f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r = fmaxf(r, red[w]);
    *out = r;
  }
}
// per-column max |Y[:, c0 + c]| as float bits (non-negative floats order like uint)
__global__ void k_col_amax(const float *Y, long long M, int N, int c0, int nc, unsigned int *out) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= nc) return;
  float m = 0.0f;
  for (long long r = blockIdx.y; r < M; r += gridDim.y) m = fmaxf(m, fabsf(Y[r * N + c0 + c]));
  atomicMax(out + c, __float_as_uint(m));
}
__global__ void k_exp_conv_in(const unsigned int *amax_bits, const float *conv_b,
                              const int32_t *e_w, int cc, int32_t *e_u, int32_t *bq) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= cc) return;
  const int e = pot_exponent((double)__uint_as_float(amax_bits[c]), 127.0);
  e_u[c] = e;
  double v = rint(ldexp((double)conv_b[c], -(e_w[c] + e)));
  v = fmin(fmax(v, -2147483647.0), 2147483647.0);
  bq[c] = (int32_t)v;
}
// conv output exponents from max |SiLU| per channel (single CTA)
__global__ void k_exp_conv_out(const unsigned int *amax, int di, int hd, int ds, int32_t *exps,
                               fm_exp_layout X) {
  const int nh = di / hd, cc = di + 2 * ds;
  for (int h = threadIdx.x; h < nh + 2; h += blockDim.x) {
    const int lo = h < nh ? h * hd : (h == nh ? di : di + ds);
    const int n = h < nh ? hd : ds;
    unsigned int m = 0;
    for (int c = lo; c < lo + n; ++c) m = amax[c] > m ? amax[c] : m;
    const int e = pot_exponent((double)m, 127.0) - 16;
    if (h < nh) exps[X.e_x + h] = e;
    else if (h == nh) exps[X.e_B] = e;
    else exps[X.e_C] = e;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < cc; c += blockDim.x)
    exps[X.e_o + c] = c < di ? exps[X.e_x + c / hd] : (c < di + ds ? exps[X.e_B] : exps[X.e_C]);
}
// headroom: 2^29 of the 31-bit state's 2^30 clamp, 2^14 of the 16-bit one's 2^15
__global__ void k_exp_state(const unsigned long long *amax_h, int nh, int32_t *exps,
                            fm_exp_layout X, double headroom) {
  const int h = threadIdx.x;
  if (h >= nh) return;
  const int ef = exps[X.e_x + h] + exps[X.e_B] - 15;
  const int e = pot_exponent((double)amax_h[h], headroom) + ef;
  exps[X.e_h + h] = e > ef ? e : ef;
}
__global__ void k_exp_y(const unsigned long long *ystat, int nh, int32_t *exps, fm_exp_layout X) {
  const int h = threadIdx.x;
  if (h >= nh) return;
  const int a = exps[X.e_C] + exps[X.e_h + h], b = exps[X.e_D + h] + exps[X.e_x + h];
  const int ef = a < b ? a : b, hi = a > b ? a : b;
  const int e = pot_exponent((double)ystat[h], 536870912.0) + ef;
  exps[X.e_y + h] = e > hi - 16 ? e : hi - 16;
}
// e_g: before the statistics pass (gstat == null) the lower bound max e_y - 16
// (every gate shift >= 0), after it the calibrated value.
__global__ void k_exp_gate(const unsigned long long *gstat, int nh, int32_t *exps,
                           fm_exp_layout X) {
  if (threadIdx.x != 0) return;
  int ymax = -1000000;
  for (int h = 0; h < nh; ++h) ymax = exps[X.e_y + h] > ymax ? exps[X.e_y + h] : ymax;
  int e = ymax - 16;
  if (gstat)
    for (int h = 0; h < nh; ++h) {
      const int eh = pot_exponent((double)gstat[h], 32767.0) + exps[X.e_y + h] - 16;
      e = eh > e ? eh : e;
    }
  exps[X.e_g] = e;
}

namespace {
struct CalibWs {
  MixerWs m;
  float *Y;               // [M, n_in] in_proj output (fp32)
  float *amax_row;        // [M]
  unsigned int *col_amax; // [cc]
  unsigned int *silu_amax;// [cc]
  unsigned long long *stat;  // [nh]
};
CalibWs carve_calib(Carver &c, const Dims &d, int B, int T) {
  const long long M = (long long)B * T;
  CalibWs w;
  w.m = carve_mixer(c, d, B, T);
  w.Y = c.take<float>(M * d.n_in);
  w.amax_row = c.take<float>(M);
  w.col_amax = c.take<unsigned int>(d.cc);
  w.silu_amax = c.take<unsigned int>(d.cc);
  w.stat = c.take<unsigned long long>(d.nh);
  return w;
}
}  // namespace

extern "C" size_t fm_calib_workspace_bytes(const fm_shape *shape, int B, int T) {
  Dims d;
  if (check_shape(shape, &d, __func__) != FM_OK || B < 0 || T < 0) return 0;
  Carver c{nullptr, 0};
  carve_calib(c, d, B, T);
  return c.off + 256;
}

extern "C" fm_status fm_calibrate_layer(const fm_layer *L, const float *conv_b, int32_t *exps,
                                        int32_t *conv_bq, float *static_amax, const float *xcal,
                                        int B, int T, int residual, float *out, void *ws,
                                        size_t ws_bytes, fm_stream stream) {
  Dims d;
  FM_TRY(check_layer(L, &d, __func__));
  NEED(conv_b);
  NEED(exps);
  NEED(conv_bq);
  NEED(static_amax);
  NEED(xcal);
  NEED(out);
  if (exps != L->exps || conv_bq != L->conv_bq || static_amax != L->static_amax)
    return fail(FM_ERR_INVALID_ARG, "fm_calibrate_layer: table pointers must be the layer's own");
  if (B <= 0 || T <= 0) return fail(FM_ERR_SHAPE, "fm_calibrate_layer: need B, T > 0");
  FM_TRY(check_batch(B, T, __func__));
  const size_t need = fm_calib_workspace_bytes(&L->shape, B, T);
  if (!ws || ws_bytes < need || !aligned16(ws))
    return fail(FM_ERR_WORKSPACE, "fm_calibrate_layer: workspace needs %zu bytes", need);
  cudaStream_t s = (cudaStream_t)stream;
  const long long M = (long long)B * T;
  const fm_exp_layout X = fm_exp_table_layout(&L->shape);
  Carver c{reinterpret_cast<uint8_t *>(ws), 0};
  const CalibWs w = carve_calib(c, d, B, T);
  const MixerWs &m = w.m;

  // 1. in_proj input: max |rotated (normed) input| -> static_amax[0]
  FM_TRY(launch_hadamard_quant(xcal, M, d.dm, L->prenorm_w, L->rotate, FM_DYNAMIC, nullptr, m.q_in,
                               m.sx_in, w.amax_row, s));
  k_max_f32<<<1, 1024, 0, s>>>(w.amax_row, M, static_amax);
  FM_TRY(launched("k_max_f32"));
  if (L->mode == FM_STATIC)
    FM_TRY(launch_hadamard_quant(xcal, M, d.dm, L->prenorm_w, L->rotate, FM_STATIC, static_amax,
                                 m.q_in, m.sx_in, nullptr, s));
  // 2. conv input exponents from the dequantised in_proj output; bias codes
  FM_TRY(launch_gemm(m.q_in, M, L->w_in_q, d.n_in, d.dm,
                     plain_epilogue(M, d.n_in, m.sx_in, L->w_in_s, nullptr, w.Y, nullptr), s));
  FM_CHECK_CUDA(cudaMemsetAsync(w.col_amax, 0, sizeof(unsigned int) * d.cc, s));
  {
    const long long gy = M < 1024 ? M : 1024;
    k_col_amax<<<dim3((d.cc + 127) / 128, (unsigned)gy), 128, 0, s>>>(w.Y, M, d.n_in, d.di, d.cc,
                                                                       w.col_amax);
    FM_TRY(launched("k_col_amax"));
  }
  k_exp_conv_in<<<(d.cc + 127) / 128, 128, 0, s>>>(w.col_amax, conv_b, exps + X.e_w, d.cc,
                                                   exps + X.e_u, conv_bq);
  FM_TRY(launched("k_exp_conv_in"));
  FM_TRY(in_proj_impl(m.q_in, m.sx_in, M, L->w_in_q, L->w_in_s, d, exps + X.e_u, m.z, m.xbc, m.dt,
                      s));
  // 3. conv output exponents (statistics pass with e_o = 0, then the real pass)
  k_calib_fill<<<(d.cc + 127) / 128, 128, 0, s>>>(exps + X.e_o, d.cc, 0);
  FM_TRY(launched("k_calib_fill"));
  FM_CHECK_CUDA(cudaMemsetAsync(w.silu_amax, 0, sizeof(unsigned int) * d.cc, s));
  FM_TRY(launch_conv(m.xbc, B, T, d.cc, L->conv_wq, conv_bq, exps, nullptr, m.xo, w.silu_amax, s));
  k_exp_conv_out<<<1, 256, 0, s>>>(w.silu_amax, d.di, d.hd, d.ds, exps, X);
  FM_TRY(launched("k_exp_conv_out"));
  FM_TRY(launch_conv(m.xbc, B, T, d.cc, L->conv_wq, conv_bq, exps, nullptr, m.xo, nullptr, s,
                     m.e_tok, &d));
  // 4. state exponent: 64-bit run at the finest exponent
  FM_CHECK_CUDA(cudaMemsetAsync(w.stat, 0, sizeof(unsigned long long) * d.nh, s));
  FM_TRY(launch_scan<2>(scan_args(d, m.xo, m.dt, T, L->dt_bias, L->A_q, L->D_q, exps, X, nullptr,
                                  m.y, w.stat, m.e_tok),
                        B, s));
  k_exp_state<<<1, 128, 0, s>>>(w.stat, d.nh, exps, X, state16() ? 16384.0 : 536870912.0);
  FM_TRY(launched("k_exp_state"));
  // 5. output exponent: max |y| at the finer term exponent
  FM_CHECK_CUDA(cudaMemsetAsync(w.stat, 0, sizeof(unsigned long long) * d.nh, s));
  FM_TRY(launch_scan<1>(scan_args(d, m.xo, m.dt, T, L->dt_bias, L->A_q, L->D_q, exps, X, nullptr,
                                  m.y, w.stat, m.e_tok),
                        B, s));
  k_exp_y<<<1, 128, 0, s>>>(w.stat, d.nh, exps, X);
  FM_TRY(launched("k_exp_y"));
  FM_TRY(launch_scan_v2(scan_args(d, m.xo, m.dt, T, L->dt_bias, L->A_q, L->D_q, exps, X, nullptr,
                                  m.y, nullptr, m.e_tok),
                        B, m.scan, s));
  // 6. gate exponent, then the out_proj input amax
  k_exp_gate<<<1, 32, 0, s>>>(nullptr, d.nh, exps, X);
  FM_TRY(launched("k_exp_gate"));
  FM_CHECK_CUDA(cudaMemsetAsync(w.stat, 0, sizeof(unsigned long long) * d.nh, s));
  FM_TRY(gate_impl(m.y, m.z, M, d, exps, X, L->norm_w, L->rotate, FM_DYNAMIC, nullptr, m.q_out,
                   m.sx_out, nullptr, w.stat, nullptr, s));
  k_exp_gate<<<1, 32, 0, s>>>(w.stat, d.nh, exps, X);
  FM_TRY(launched("k_exp_gate"));
  FM_TRY(gate_impl(m.y, m.z, M, d, exps, X, L->norm_w, L->rotate, FM_DYNAMIC, nullptr, m.q_out,
                   m.sx_out, w.amax_row, nullptr, nullptr, s));
  k_max_f32<<<1, 1024, 0, s>>>(w.amax_row, M, static_amax + 1);
  FM_TRY(launched("k_max_f32"));
  if (L->mode == FM_STATIC)
    FM_TRY(gate_impl(m.y, m.z, M, d, exps, X, L->norm_w, L->rotate, FM_STATIC, static_amax + 1,
                     m.q_out, m.sx_out, nullptr, nullptr, nullptr, s));
  // 7. the layer's output on the calibration set
  return launch_gemm(m.q_out, M, L->w_out_q, d.dm, d.di,
                     plain_epilogue(M, d.dm, m.sx_out, L->w_out_s, residual ? xcal : nullptr, out,
                                    nullptr),
                     s);
}
