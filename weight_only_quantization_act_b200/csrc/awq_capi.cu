// awq_capi.cu - host side of libawq: argument validation, workspace layout, TMA descriptors and the
// launch sequence of every entry point declared in include/awq.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "awq.h"
#include "kernel_loss_gemm.cuh"
#include "kernel_w4a16.cuh"
#include "kernel_w4a16_decode.cuh"
#include "kernels_simple.cuh"

namespace {

thread_local char g_err[512] = "";
thread_local cudaEvent_t g_prof_before = nullptr;
thread_local cudaEvent_t g_prof_after = nullptr;
std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};

awq_status fail(awq_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

awq_status ok() {
  g_err[0] = '\0';
  return AWQ_OK;
}

#define AWQ_CUDA(call)                                                                        \
  do {                                                                                        \
    cudaError_t e_ = (call);                                                                  \
    if (e_ != cudaSuccess) return fail(AWQ_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

struct DeviceInfo {
  unsigned long long ctx_id = 0;  // CUDA context the cached state below belongs to
  int sms = 0;
  int cc_major = 0;
  bool gemm_attr_set = false;
  int gemm_clusters = 0;  // CTA pairs of the loss GEMM that fit on the device at once
  int w4_clusters = 0;    // CTA pairs of the W4A16 GEMM that fit on the device at once
};

constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

using PFN_ctx_get_current = CUresult (*)(CUcontext*);
using PFN_ctx_get_id = CUresult (*)(CUcontext, unsigned long long*);

template <typename F>
F driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion(name, &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<F>(p);
}

// The current device and the unique id of its current CUDA context. Per-device state cached by this
// file (function attributes, the no-alloc scratch address) belongs to one context: after cudaDeviceReset
// the primary context is created anew, the library's device code is loaded into it again, and the
// cached state must be rebuilt. cudaSetDevice on the current device makes its primary context current
// (creating it if needed) without allocating anything.
awq_status current_context(int* dev, unsigned long long* ctx_id) {
  static PFN_ctx_get_current get_current = nullptr;
  static PFN_ctx_get_id get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    get_current = driver_fn<PFN_ctx_get_current>("cuCtxGetCurrent");
    get_id = driver_fn<PFN_ctx_get_id>("cuCtxGetId");
  });
  AWQ_CUDA(cudaGetDevice(dev));
  if (*dev < 0 || *dev >= kMaxDevices) return fail(AWQ_ERR_UNSUPPORTED, "device index %d out of range", *dev);
  AWQ_CUDA(cudaSetDevice(*dev));
  if (get_current == nullptr || get_id == nullptr)
    return fail(AWQ_ERR_CUDA, "cuCtxGetCurrent / cuCtxGetId not available from the driver");
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
    return fail(AWQ_ERR_CUDA, "no current CUDA context on device %d", *dev);
  if (get_id(ctx, ctx_id) != CUDA_SUCCESS) return fail(AWQ_ERR_CUDA, "cuCtxGetId failed on device %d", *dev);
  return AWQ_OK;
}

awq_status device_info(DeviceInfo** out) {
  int dev = 0;
  unsigned long long ctx_id = 0;
  {
    awq_status s = current_context(&dev, &ctx_id);
    if (s != AWQ_OK) return s;
  }
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.ctx_id != ctx_id) d = DeviceInfo{};  // a new context: attributes are set again
  if (d.sms == 0) {
    d.ctx_id = ctx_id;
    AWQ_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
    AWQ_CUDA(cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev));
  }
  if (d.cc_major != 10)
    return fail(AWQ_ERR_UNSUPPORTED, "compute capability %d.x: this library is built for sm_100a", d.cc_major);
  if (!d.gemm_attr_set) {
    AWQ_CUDA(cudaFuncSetAttribute(awq::lg::loss_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  awq::lg::SMEM_BYTES));
    AWQ_CUDA(cudaFuncSetAttribute(awq::quantize_pack_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  awq::kPackSmemBytes));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(d.sms & ~1));
    cfg.blockDim = dim3(awq::lg::THREADS);
    cfg.dynamicSmemBytes = awq::lg::SMEM_BYTES;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    AWQ_CUDA(cudaOccupancyMaxActiveClusters(&d.gemm_clusters, awq::lg::loss_gemm_kernel, &cfg));
    if (d.gemm_clusters < 1) return fail(AWQ_ERR_UNSUPPORTED, "the loss GEMM does not fit on this device");
    AWQ_CUDA(cudaFuncSetAttribute(awq::dq::w4a16_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  awq::dq::SMEM_BYTES));
    cfg.blockDim = dim3(awq::dq::THREADS);
    cfg.dynamicSmemBytes = awq::dq::SMEM_BYTES;
    AWQ_CUDA(cudaOccupancyMaxActiveClusters(&d.w4_clusters, awq::dq::w4a16_gemm_kernel, &cfg));
    if (d.w4_clusters < 1) return fail(AWQ_ERR_UNSUPPORTED, "the W4A16 GEMM does not fit on this device");
    AWQ_CUDA(cudaFuncSetAttribute(awq::dec::w4a16_decode_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  awq::dec::Shape<16>::SMEM));
    AWQ_CUDA(cudaFuncSetAttribute(awq::dec::w4a16_decode_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  awq::dec::Shape<32>::SMEM));
    AWQ_CUDA(cudaFuncSetAttribute(awq::dec::w4a16_decode_kernel<48>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  awq::dec::Shape<48>::SMEM));
    AWQ_CUDA(cudaFuncSetAttribute(awq::dec::w4a16_decode_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  awq::dec::Shape<64>::SMEM));
    d.gemm_attr_set = true;
  }
  *out = &d;
  return AWQ_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Row-major bf16 [rows, cols] with row stride ld (elements), tiles of box_rows x 64 columns, 128 B swizzle.
awq_status make_tmap(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld, int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return fail(AWQ_ERR_CUDA, "cuTensorMapEncodeTiled not available from the driver");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(awq::lg::BK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(AWQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
  return AWQ_OK;
}

// Generic row-major 2-D map without swizzle: [rows][cols] of elements of `esize` bytes.
awq_status make_tmap_plain(CUtensorMap* map, const void* base, CUtensorMapDataType type, int esize, int64_t rows,
                           int64_t cols, int64_t ld, int box_cols, int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return fail(AWQ_ERR_CUDA, "cuTensorMapEncodeTiled not available from the driver");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * static_cast<cuuint64_t>(esize)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(AWQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
  return AWQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Code words [rows][cols] (uint32) in boxes of 32 words x box_rows with 128-byte swizzle.
awq_status make_tmap_codes_sw128(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return fail(AWQ_ERR_CUDA, "cuTensorMapEncodeTiled not available from the driver");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 4};
  cuuint32_t box[2] = {32u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(AWQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
  return AWQ_OK;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ----------------------------------------------------------------------------- workspace layouts
struct ActLayout {
  int n_chunks;
  size_t bytes;
};
ActLayout act_layout(int64_t N, int64_t K) {
  ActLayout l;
  l.n_chunks = static_cast<int>((N + awq::kActChunk - 1) / awq::kActChunk);
  l.bytes = align_up(static_cast<size_t>(l.n_chunks) * static_cast<size_t>(K) * sizeof(double), 256);
  return l;
}

struct ScaleLayout {
  int nblk;
  size_t part_off, bytes;
};
ScaleLayout scale_layout(int64_t K, int n_grid) {
  ScaleLayout l;
  l.nblk = static_cast<int>((K + awq::kScaleThreads - 1) / awq::kScaleThreads);
  l.part_off = 0;
  l.bytes = align_up(static_cast<size_t>(n_grid) * l.nblk * sizeof(float2), 256);
  return l;
}

struct SearchLayout {
  int64_t O_pad, tiles_n, tiles_o;
  size_t status_off, produced_off, table_off, rtable_off, spart_off, wmean_off, wpart_off, rowstep_off, partials_off,
      dw_off, bytes;
  ScaleLayout sl;
};
SearchLayout search_layout(int64_t N, int64_t K, int64_t O, int n_grid) {
  SearchLayout l;
  l.O_pad = (O + awq::lg::BN - 1) / awq::lg::BN * awq::lg::BN;
  l.tiles_n = (N + awq::lg::BM - 1) / awq::lg::BM;
  l.tiles_o = l.O_pad / awq::lg::BN;
  l.sl = scale_layout(K, n_grid);
  size_t off = 0;
  l.status_off = off;  // DeviceStatus (16 B), finalize block counter (4 B), tile counter (4 B)
  l.produced_off = off + 256;      // unsigned produced[AWQ_MAX_N_GRID]
  off += 512;
  l.table_off = off;
  off = align_up(off + static_cast<size_t>(n_grid) * K * sizeof(float), 256);
  l.rtable_off = off;
  off = align_up(off + static_cast<size_t>(n_grid) * K * sizeof(float), 256);
  l.spart_off = off;
  off = align_up(off + l.sl.bytes, 256);
  l.wmean_off = off;  // weight-aware rule: mean |W| per column and its fixed-order chunk sums
  off = align_up(off + static_cast<size_t>(K) * sizeof(float), 256);
  l.wpart_off = off;
  off = align_up(off + act_layout(O, K).bytes, 256);
  l.rowstep_off = off;  // INT8 quantizer: per-candidate, per-row steps
  off = align_up(off + static_cast<size_t>(n_grid) * l.O_pad * sizeof(float), 256);
  l.partials_off = off;
  off = align_up(off + static_cast<size_t>(n_grid) * l.tiles_o * l.tiles_n * awq::lg::PARTIALS_PER_TILE *
                           sizeof(double), 1024);
  l.dw_off = off;
  off = align_up(off + static_cast<size_t>(n_grid) * l.O_pad * K * 2, 1024);
  l.bytes = off;
  return l;
}

awq_status check_group(int group) {
  if (group != 128) return fail(AWQ_ERR_UNSUPPORTED, "group size %d: only 128 is supported", group);
  return AWQ_OK;
}

awq_status check_grid(int n_grid) {
  if (n_grid < 1 || n_grid > AWQ_MAX_N_GRID)
    return fail(AWQ_ERR_INVALID_ARG, "n_grid %d outside [1, %d]", n_grid, AWQ_MAX_N_GRID);
  return AWQ_OK;
}

awq_status check_matrix(const char* name, const void* p, int64_t rows, int64_t K, int64_t ld) {
  if (p == nullptr) return fail(AWQ_ERR_INVALID_ARG, "%s is null", name);
  if (!aligned16(p)) return fail(AWQ_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  if (rows < 1 || K < 1) return fail(AWQ_ERR_INVALID_ARG, "%s has an empty shape (%lld x %lld)", name,
                                     static_cast<long long>(rows), static_cast<long long>(K));
  if (rows >= (1ll << 31) || K >= (1ll << 31)) return fail(AWQ_ERR_INVALID_ARG, "%s is too large", name);
  if (ld < K || ld % 8 != 0)
    return fail(AWQ_ERR_INVALID_ARG, "%s row stride %lld must be >= K (%lld) and a multiple of 8", name,
                static_cast<long long>(ld), static_cast<long long>(K));
  return AWQ_OK;
}

// The interface bounds the statistic's rows by 65535 chunks of 256 (N <= 16,776,960).
awq_status check_act_chunks(const char* name, int64_t rows) {
  const int64_t n_chunks = (rows + awq::kActChunk - 1) / awq::kActChunk;
  if (n_chunks > 65535)
    return fail(AWQ_ERR_INVALID_ARG, "%s has %lld rows: at most 65535 chunks of %d (%lld rows) are supported", name,
                static_cast<long long>(rows), awq::kActChunk, 65535ll * awq::kActChunk);
  return AWQ_OK;
}

awq_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(AWQ_ERR_CUDA, "launch of %s failed: %s", what, cudaGetErrorString(e));
  return AWQ_OK;
}

// Column sums of |A| (rows x K, stride ld) in the statistic's fixed order, then their means: a chunk-sum
// kernel over (chunk, column block) work items, as many CTAs as make every CTA take the same number of
// items within the resident CTAs of the device, then the finaliser over the fp64 partial array part. Layers
// with fewer than four 512-column items per SM take the narrow kernel (256-column items, more rows in
// flight per thread).
awq_status launch_act_stats(const void* A, int64_t rows, int64_t K, int64_t ld, double* part, float* mean, int sms,
                            cudaStream_t st) {
  const int64_t n_chunks = (rows + awq::kActChunk - 1) / awq::kActChunk;
  const int64_t wide_items = n_chunks * ((K + awq::kActColsPerBlock - 1) / awq::kActColsPerBlock);
  const bool narrow = wide_items < 4ll * sms;
  const int64_t items = narrow ? n_chunks * ((K + awq::kActNarrowColsPerBlock - 1) / awq::kActNarrowColsPerBlock)
                               : wide_items;
  const int64_t resident = static_cast<int64_t>(sms) * (narrow ? awq::kActNarrowCtasPerSm : awq::kActCtasPerSm);
  const int64_t per_cta = (items + resident - 1) / resident;
  const int64_t ctas = (items + per_cta - 1) / per_cta;
  if (narrow)
    awq::act_chunk_sums_narrow_kernel<<<static_cast<unsigned>(ctas), awq::kActNarrowThreads, 0, st>>>(
        static_cast<const uint16_t*>(A), rows, K, ld, part);
  else
    awq::act_chunk_sums_kernel<<<static_cast<unsigned>(ctas), awq::kActThreads, 0, st>>>(
        static_cast<const uint16_t*>(A), rows, K, ld, part);
  {
    awq_status s = check_launch("act_chunk_sums_kernel");
    if (s != AWQ_OK) return s;
  }
  awq::act_finalize_kernel<<<static_cast<unsigned>((K + awq::kActFinalizeThreads - 1) / awq::kActFinalizeThreads),
                             awq::kActFinalizeThreads, 0, st>>>(part, rows, K, static_cast<int>(n_chunks), mean);
  return check_launch("act_finalize_kernel");
}

#define AWQ_TRY(x)                      \
  do {                                  \
    awq_status s_ = (x);                \
    if (s_ != AWQ_OK) return s_;        \
  } while (0)

awq_status launch_scale_table(const float* act, const float* wmean, int64_t K, int n_grid, int mode, bool exact_pow,
                              float* table, float* rtable, float2* part, cudaStream_t st) {
  const int nblk = static_cast<int>((K + awq::kScaleThreads - 1) / awq::kScaleThreads);
  dim3 grid(nblk, n_grid);
  awq::scale_pow_kernel<<<grid, awq::kScaleThreads, 0, st>>>(act, wmean, K, n_grid, mode, exact_pow ? 1 : 0, table,
                                                              part);
  AWQ_TRY(check_launch("scale_pow_kernel"));
  awq::scale_normalize_kernel<<<grid, awq::kScaleThreads, 0, st>>>(table, rtable, part, K, nblk, mode);
  return check_launch("scale_normalize_kernel");
}

// Tile raster of the loss GEMM: a group of dW bands advances together over the token blocks, so each
// X tile is read from DRAM once per group while the group's bands (256 rows x K each) are re-read by
// every token block. In flight, the pairs sit at spread-out points of their K loops, so the bands stay
// in L2 only if the whole group (bands x 512 K bytes) fits in about half of it; beyond that they are
// fetched again and again (measured on B200 at K = 28672: 4 bands 1.08 GHz under the power cap, 8
// bands 1.02 GHz, 16 bands 0.88 GHz). Fewer bands mean more X reads, so take as many as fit, at most 8.
int loss_bands_per_group(int64_t K) {
  const int64_t band_bytes = static_cast<int64_t>(awq::lg::BN) * K * 2;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(8, (60ll << 20) / band_bytes)));
}

int scale_mode_of(unsigned flags) {
  if (flags & AWQ_FLAG_SCALES_WEIGHT_AWARE) return awq::kScalesWeightAware;
  if (flags & AWQ_FLAG_SCALES_RMS) return awq::kScalesRms;
  return awq::kScalesP4;
}

}  // namespace

extern "C" {

const char* awq_last_error(void) { return g_err; }

int awq_version(void) { return 100; }

void awq_set_profile_events(void* before_loss_gemm, void* after_loss_gemm) {
  g_prof_before = static_cast<cudaEvent_t>(before_loss_gemm);
  g_prof_after = static_cast<cudaEvent_t>(after_loss_gemm);
}

void awq_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns < 1000000ull ? 1000000ull : ns); }

size_t awq_act_stats_workspace_size(int64_t N, int64_t K) {
  if (N < 1 || K < 1) return 0;
  return act_layout(N, K).bytes;
}

awq_status awq_act_stats(const void* X, int64_t N, int64_t K, int64_t ldx, void* workspace, size_t ws_bytes,
                         float* act_mean, awq_stream_t stream) {
  AWQ_TRY(check_matrix("X", X, N, K, ldx));
  if (K % 2 != 0) return fail(AWQ_ERR_INVALID_ARG, "K must be even");
  if (act_mean == nullptr) return fail(AWQ_ERR_INVALID_ARG, "act_mean is null");
  AWQ_TRY(check_act_chunks("X", N));
  const ActLayout l = act_layout(N, K);
  if (workspace == nullptr || ws_bytes < l.bytes)
    return fail(AWQ_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", l.bytes, workspace ? ws_bytes : 0);
  if (!aligned16(workspace)) return fail(AWQ_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
  DeviceInfo* d = nullptr;
  AWQ_TRY(device_info(&d));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  double* part = static_cast<double*>(workspace);
  AWQ_TRY(launch_act_stats(X, N, K, ldx, part, act_mean, d->sms, st));
  return ok();
}

size_t awq_scale_table_workspace_size(int64_t K, int n_grid) {
  if (K < 1 || n_grid < 1 || n_grid > AWQ_MAX_N_GRID) return 0;
  return scale_layout(K, n_grid).bytes;
}

awq_status awq_scale_table_ex(const float* act_mean, const float* weight_mean, int64_t K, int n_grid, unsigned flags,
                              void* workspace, size_t ws_bytes, float* table, awq_stream_t stream) {
  if (act_mean == nullptr || table == nullptr) return fail(AWQ_ERR_INVALID_ARG, "null pointer");
  if (K < 1 || K >= (1ll << 31)) return fail(AWQ_ERR_INVALID_ARG, "bad K");
  AWQ_TRY(check_grid(n_grid));
  if (flags & ~(AWQ_FLAG_EXACT_POW | AWQ_FLAG_SCALES_WEIGHT_AWARE | AWQ_FLAG_SCALES_RMS))
    return fail(AWQ_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if ((flags & AWQ_FLAG_SCALES_WEIGHT_AWARE) && (flags & AWQ_FLAG_SCALES_RMS))
    return fail(AWQ_ERR_INVALID_ARG, "choose one candidate-scale rule");
  if ((flags & AWQ_FLAG_SCALES_WEIGHT_AWARE) && weight_mean == nullptr)
    return fail(AWQ_ERR_INVALID_ARG, "the weight-aware rule needs weight_mean");
  const ScaleLayout l = scale_layout(K, n_grid);
  if (workspace == nullptr || ws_bytes < l.bytes)
    return fail(AWQ_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", l.bytes, workspace ? ws_bytes : 0);
  DeviceInfo* d = nullptr;
  AWQ_TRY(device_info(&d));
  AWQ_TRY(launch_scale_table(act_mean, weight_mean, K, n_grid, scale_mode_of(flags), (flags & AWQ_FLAG_EXACT_POW) != 0,
                             table, nullptr, reinterpret_cast<float2*>(static_cast<char*>(workspace) + l.part_off),
                             reinterpret_cast<cudaStream_t>(stream)));
  return ok();
}

awq_status awq_scale_table(const float* act_mean, int64_t K, int n_grid, unsigned flags, void* workspace,
                           size_t ws_bytes, float* table, awq_stream_t stream) {
  if (flags & AWQ_FLAG_SCALES_WEIGHT_AWARE)
    return fail(AWQ_ERR_INVALID_ARG, "the weight-aware rule needs awq_scale_table_ex");
  return awq_scale_table_ex(act_mean, nullptr, K, n_grid, flags, workspace, ws_bytes, table, stream);
}

size_t awq_search_workspace_size(int64_t N, int64_t K, int64_t O, int group, int n_grid) {
  if (N < 1 || K < 1 || O < 1 || (group != 128 && group != 0) || n_grid < 1 || n_grid > AWQ_MAX_N_GRID) return 0;
  return search_layout(N, K, O, n_grid).bytes;
}

awq_status awq_search_get_layout(int64_t N, int64_t K, int64_t O, int group, int n_grid, awq_search_layout* out) {
  if (out == nullptr) return fail(AWQ_ERR_INVALID_ARG, "out is null");
  if (group != 0) AWQ_TRY(check_group(group));
  AWQ_TRY(check_grid(n_grid));
  if (N < 1 || K < 1 || O < 1) return fail(AWQ_ERR_INVALID_ARG, "empty shape");
  const SearchLayout l = search_layout(N, K, O, n_grid);
  out->tile_n = awq::lg::BM;
  out->tile_o = awq::lg::BN;
  out->tiles_n = l.tiles_n;
  out->tiles_o = l.tiles_o;
  out->partials_per_tile = awq::lg::PARTIALS_PER_TILE;
  out->partials_offset = l.partials_off;
  out->workspace_bytes = l.bytes;
  return ok();
}

awq_status awq_search_ex(const void* X, int64_t N, int64_t K, int64_t ldx, const void* W, int64_t O, int64_t ldw,
                         const float* act_mean, int group, int n_grid, unsigned flags, void* workspace,
                         size_t ws_bytes, double* losses, int* best_j, float* scales, awq_stream_t stream) {
  const bool int8 = (flags & AWQ_FLAG_QUANT_INT8) != 0;
  if (int8 && group != 0)
    return fail(AWQ_ERR_UNSUPPORTED, "group %d: the INT8 quantizer is per channel (pass group 0)", group);
  if (!int8) AWQ_TRY(check_group(group));
  AWQ_TRY(check_grid(n_grid));
  AWQ_TRY(check_matrix("X", X, N, K, ldx));
  AWQ_TRY(check_matrix("W", W, O, K, ldw));
  if (K % 128 != 0) return fail(AWQ_ERR_INVALID_ARG, "K (%lld) must be a multiple of 128", static_cast<long long>(K));
  if (act_mean == nullptr || losses == nullptr || best_j == nullptr || scales == nullptr)
    return fail(AWQ_ERR_INVALID_ARG, "null output or act_mean pointer");
  if (flags & ~(AWQ_FLAG_EXACT_DIVISION | AWQ_FLAG_EXACT_POW | AWQ_FLAG_INJECT_STALL | AWQ_FLAG_SCALES_WEIGHT_AWARE |
                AWQ_FLAG_SCALES_RMS | AWQ_FLAG_QUANT_INT8))
    return fail(AWQ_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  if ((flags & AWQ_FLAG_SCALES_WEIGHT_AWARE) && (flags & AWQ_FLAG_SCALES_RMS))
    return fail(AWQ_ERR_INVALID_ARG, "choose one candidate-scale rule");
  if (flags & AWQ_FLAG_SCALES_WEIGHT_AWARE) AWQ_TRY(check_act_chunks("W", O));  // mean |W| per column
  const SearchLayout l = search_layout(N, K, O, n_grid);
  if (static_cast<int64_t>(n_grid) * l.O_pad >= (1ll << 31))
    return fail(AWQ_ERR_INVALID_ARG, "n_grid * O is too large");
  if (static_cast<int64_t>(n_grid) * l.tiles_o * l.tiles_n >= (1ll << 31))
    return fail(AWQ_ERR_INVALID_ARG, "too many tiles");
  if (workspace == nullptr || ws_bytes < l.bytes)
    return fail(AWQ_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", l.bytes, workspace ? ws_bytes : 0);
  if ((reinterpret_cast<uintptr_t>(workspace) & 1023u) != 0)
    return fail(AWQ_ERR_INVALID_ARG, "workspace must be 1024-byte aligned");
  DeviceInfo* d = nullptr;
  AWQ_TRY(device_info(&d));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  auto* status = reinterpret_cast<awq::DeviceStatus*>(ws + l.status_off);
  float* table = reinterpret_cast<float*>(ws + l.table_off);
  float* rtable = reinterpret_cast<float*>(ws + l.rtable_off);
  auto* spart = reinterpret_cast<float2*>(ws + l.spart_off);
  auto* partials = reinterpret_cast<double*>(ws + l.partials_off);
  auto* dw = reinterpret_cast<__nv_bfloat16*>(ws + l.dw_off);

  CUtensorMap tmX, tmD;
  AWQ_TRY(make_tmap(&tmX, X, N, K, ldx, awq::lg::HALF));
  AWQ_TRY(make_tmap(&tmD, dw, static_cast<int64_t>(n_grid) * l.O_pad, K, K, awq::lg::HALF));
  auto* produced = reinterpret_cast<unsigned int*>(ws + l.produced_off);

  AWQ_CUDA(cudaMemsetAsync(ws + l.status_off, 0, 512, st));  // status word and production counters
  const int mode = scale_mode_of(flags);
  float* wmean = reinterpret_cast<float*>(ws + l.wmean_off);
  if (mode == awq::kScalesWeightAware) {
    // mean |W| per column: the activation statistic's fixed-order kernels run on W
    double* wpart = reinterpret_cast<double*>(ws + l.wpart_off);
    AWQ_TRY(launch_act_stats(W, O, K, ldw, wpart, wmean, d->sms, st));
  }
  AWQ_TRY(launch_scale_table(act_mean, wmean, K, n_grid, mode, (flags & AWQ_FLAG_EXACT_POW) != 0, table, rtable, spart,
                             st));
  float* rowstep = nullptr;
  if (int8) {
    // The per-channel step needs the whole row's max |w'| before any element is coded.
    rowstep = reinterpret_cast<float*>(ws + l.rowstep_off);
    dim3 rgrid(static_cast<unsigned>(l.O_pad * 32 / awq::kRowThreads), static_cast<unsigned>(n_grid));
    awq::int8_rowstep_kernel<<<rgrid, awq::kRowThreads, 0, st>>>(static_cast<const uint16_t*>(W), O, l.O_pad, K, ldw,
                                                                 table, rowstep);
    AWQ_TRY(check_launch("int8_rowstep_kernel"));
  }

  awq::lg::Params p;
  p.n_tiles_n = static_cast<int>(l.tiles_n);
  p.band_begin = 0;
  p.n_bands = static_cast<int>(static_cast<int64_t>(n_grid) * l.tiles_o);
  p.num_kb = static_cast<int>(K / awq::lg::BK);
  p.num_tiles = p.n_tiles_n * p.n_bands;
  p.bands_per_group = loss_bands_per_group(K);
  p.partials = partials;
  p.status = status;
  p.limit_ns = g_wait_limit_ns.load();
  p.flags = flags;
  p.tiles_o = static_cast<int>(l.tiles_o);
  p.n_grid = n_grid;
  p.prod.W = static_cast<const uint16_t*>(W);
  p.prod.O = O;
  p.prod.O_pad = l.O_pad;
  p.prod.K = K;
  p.prod.ldw = ldw;
  p.prod.segs = (K + awq::kProdWarpCols - 1) / awq::kProdWarpCols;
  p.prod.table = table;
  p.prod.rtable = rtable;
  p.prod.dW = dw;
  p.prod.exact = (flags & AWQ_FLAG_EXACT_DIVISION) ? 1 : 0;
  p.prod.rowstep = rowstep;
  p.items_per_cand = l.O_pad * p.prod.segs;
  p.produced = produced;
  p.tile_counter = reinterpret_cast<unsigned int*>(ws + l.status_off + 20);
  // L2 residency (126 MB on B200): X is read by every candidate band and W once per candidate; keep
  // them resident when they fit next to the streaming weight errors.
  const double x_bytes = 2.0 * static_cast<double>(N) * static_cast<double>(K);
  const double w_bytes = 2.0 * static_cast<double>(O) * static_cast<double>(K);
  p.keep_x = x_bytes <= 64.0e6 ? 1 : 0;
  p.prod.keep_w = (p.keep_x ? x_bytes : 0.0) + w_bytes <= 80.0e6 ? 1 : 0;

  // As many CTA pairs as fit at once, launched cooperatively: the TMA warps wait for rows that the
  // producer warps of every other CTA write, which is only safe when all CTAs are resident together.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * d->gemm_clusters));
  cfg.blockDim = dim3(awq::lg::THREADS);
  cfg.dynamicSmemBytes = awq::lg::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (g_prof_before != nullptr) AWQ_CUDA(cudaEventRecord(g_prof_before, st));
  AWQ_CUDA(cudaLaunchKernelEx(&cfg, awq::lg::loss_gemm_kernel, tmX, tmD, p));
  AWQ_TRY(check_launch("loss_gemm_kernel"));
  if (g_prof_after != nullptr) AWQ_CUDA(cudaEventRecord(g_prof_after, st));

  awq::finalize_kernel<<<n_grid, awq::kFinThreads, 0, st>>>(
      partials, l.tiles_o * l.tiles_n * awq::lg::PARTIALS_PER_TILE, n_grid,
      static_cast<double>(N) * static_cast<double>(O), table, K, losses, best_j, scales, status,
      reinterpret_cast<unsigned int*>(ws + l.status_off + 16));
  AWQ_TRY(check_launch("finalize_kernel"));
  return ok();
}

awq_status awq_search(const void* X, int64_t N, int64_t K, int64_t ldx, const void* W, int64_t O, int64_t ldw,
                      const float* act_mean, int group, int n_grid, void* workspace, size_t ws_bytes,
                      double* losses, int* best_j, float* scales, awq_stream_t stream) {
  return awq_search_ex(X, N, K, ldx, W, O, ldw, act_mean, group, n_grid, 0u, workspace, ws_bytes, losses, best_j,
                       scales, stream);
}

awq_status awq_search_status(const void* workspace, size_t ws_bytes, awq_stream_t stream) {
  if (workspace == nullptr || ws_bytes < sizeof(awq::DeviceStatus))
    return fail(AWQ_ERR_WORKSPACE, "workspace is null or too small");
  AWQ_CUDA(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  awq::DeviceStatus h;
  AWQ_CUDA(cudaMemcpy(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost));
  if (h.code == 5u)
    return fail(AWQ_ERR_TIMEOUT, "device wait gave up (site %u, block %u)", h.where, h.block);
  if (h.code != 0u) return fail(AWQ_ERR_CUDA, "unknown device status %u", h.code);
  return ok();
}

awq_status awq_quantize_pack_ex(const void* W, int64_t O, int64_t K, int64_t ldw, const float* scales, int group,
                                unsigned flags, uint32_t* codes, float* steps, float* zeros, awq_stream_t stream) {
  AWQ_TRY(check_group(group));
  AWQ_TRY(check_matrix("W", W, O, K, ldw));
  if (K % 128 != 0) return fail(AWQ_ERR_INVALID_ARG, "K (%lld) must be a multiple of 128", static_cast<long long>(K));
  if (scales == nullptr || codes == nullptr || steps == nullptr || zeros == nullptr)
    return fail(AWQ_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(scales) || !aligned16(codes))
    return fail(AWQ_ERR_INVALID_ARG, "scales and codes must be 16-byte aligned");
  if (flags & ~AWQ_FLAG_EXACT_DIVISION) return fail(AWQ_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  DeviceInfo* d = nullptr;
  AWQ_TRY(device_info(&d));
  // One resident wave of CTAs, each on one segment (1024 in-features) and 8 rows at a time: as many CTAs
  // per segment as fit, with every segment given the same number (fewer CTAs than segments: each CTA
  // walks several segments).
  const int64_t segs = (K + awq::kPackWarpCols - 1) / awq::kPackWarpCols;
  const int64_t row_octets = (O + awq::kPackThreads / 32 - 1) / (awq::kPackThreads / 32);
  const int64_t max_blocks = static_cast<int64_t>(d->sms) * awq::kPackCtasPerSm;
  int64_t blocks = std::min<int64_t>(max_blocks, row_octets * segs);
  if (blocks > segs) blocks = blocks / segs * segs;
  awq::quantize_pack_kernel<<<static_cast<unsigned>(blocks), awq::kPackThreads, awq::kPackSmemBytes,
                              reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(W), O, K, ldw, scales, (flags & AWQ_FLAG_EXACT_DIVISION) ? 1 : 0, codes, steps,
      zeros);
  AWQ_TRY(check_launch("quantize_pack_kernel"));
  return ok();
}

awq_status awq_quantize_pack(const void* W, int64_t O, int64_t K, int64_t ldw, const float* scales, int group,
                             uint32_t* codes, float* steps, float* zeros, awq_stream_t stream) {
  return awq_quantize_pack_ex(W, O, K, ldw, scales, group, 0u, codes, steps, zeros, stream);
}

awq_status awq_quantize_pack_int8(const void* W, int64_t O, int64_t K, int64_t ldw, const float* scales,
                                  unsigned flags, int8_t* codes, float* steps, awq_stream_t stream) {
  AWQ_TRY(check_matrix("W", W, O, K, ldw));
  if (K % 8 != 0) return fail(AWQ_ERR_INVALID_ARG, "K (%lld) must be a multiple of 8", static_cast<long long>(K));
  if (scales == nullptr || codes == nullptr || steps == nullptr) return fail(AWQ_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(scales) || (reinterpret_cast<uintptr_t>(codes) & 7u) != 0)
    return fail(AWQ_ERR_INVALID_ARG, "scales must be 16-byte and codes 8-byte aligned");
  if (flags & ~AWQ_FLAG_EXACT_DIVISION) return fail(AWQ_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  DeviceInfo* d = nullptr;
  AWQ_TRY(device_info(&d));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int exact = (flags & AWQ_FLAG_EXACT_DIVISION) ? 1 : 0;
  const int64_t pieces = (K + 8 * awq::kRowBlock - 1) / (8 * awq::kRowBlock);  // 16-byte pieces per thread
  if (pieces <= 16) {
    // W read once: one CTA per row with the row in registers (grid-stride over rows)
    const int64_t blocks = std::min<int64_t>(static_cast<int64_t>(d->sms) * 8, O);
    const unsigned grid = static_cast<unsigned>(blocks);
    const auto* w16 = static_cast<const uint16_t*>(W);
    if (pieces <= 1)
      awq::quantize_pack_int8_rows_kernel<1><<<grid, awq::kRowBlock, 0, st>>>(w16, O, K, ldw, scales, exact, codes, steps);
    else if (pieces <= 2)
      awq::quantize_pack_int8_rows_kernel<2><<<grid, awq::kRowBlock, 0, st>>>(w16, O, K, ldw, scales, exact, codes, steps);
    else if (pieces <= 4)
      awq::quantize_pack_int8_rows_kernel<4><<<grid, awq::kRowBlock, 0, st>>>(w16, O, K, ldw, scales, exact, codes, steps);
    else if (pieces <= 8)
      awq::quantize_pack_int8_rows_kernel<8><<<grid, awq::kRowBlock, 0, st>>>(w16, O, K, ldw, scales, exact, codes, steps);
    else
      awq::quantize_pack_int8_rows_kernel<16><<<grid, awq::kRowBlock, 0, st>>>(w16, O, K, ldw, scales, exact, codes, steps);
    AWQ_TRY(check_launch("quantize_pack_int8_rows_kernel"));
    return ok();
  }
  // very long rows: one warp per row, two passes over it (grid-stride)
  const int64_t rows_per_block = awq::kRowThreads / 32;
  const int64_t blocks = std::min<int64_t>(static_cast<int64_t>(d->sms) * 8, (O + rows_per_block - 1) / rows_per_block);
  awq::quantize_pack_int8_kernel<<<static_cast<unsigned>(blocks), awq::kRowThreads, 0, st>>>(
      static_cast<const uint16_t*>(W), O, K, ldw, scales, exact, codes, steps);
  AWQ_TRY(check_launch("quantize_pack_int8_kernel"));
  return ok();
}

}  // extern "C"

// ===================================================================================================
// Activation statistic without any allocation, for callers that cannot allocate device memory when
// they call (see awq_act_stats_noalloc in awq.h). The fp64 chunk sums live in this file-scope device
// array instead of a caller workspace. Every GPU that loads the library holds it until the process
// exits. Host code must not use the array's name as a pointer: it only names the symbol; the device
// address comes from cudaGetSymbolAddress, once per device, with that device current.
// ===================================================================================================
static __device__ __align__(256) double awq_act_scratch[AWQ_NOALLOC_SCRATCH_DOUBLES];

namespace {

struct ScratchSlot {
  bool ready = false;
  unsigned long long ctx_id = 0;  // the context the address belongs to
  double* ptr = nullptr;
};
ScratchSlot g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

// The array's device address in the current device's current context, looked up on the first call in
// that context (the device is current here, as cudaGetSymbolAddress requires).
awq_status act_scratch_address(double** out) {
  int dev = 0;
  unsigned long long ctx_id = 0;
  AWQ_TRY(current_context(&dev, &ctx_id));
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  ScratchSlot& slot = g_scratch[dev];
  if (!slot.ready || slot.ctx_id != ctx_id) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, awq_act_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(AWQ_ERR_CUDA, "cudaGetSymbolAddress of the no-alloc scratch failed on device %d: %s", dev,
                  cudaGetErrorString(e));
    slot.ptr = static_cast<double*>(p);
    slot.ctx_id = ctx_id;
    slot.ready = true;
  }
  *out = slot.ptr;
  return AWQ_OK;
}

}  // namespace

extern "C" awq_status awq_act_stats_noalloc(const void* X, int64_t N, int64_t K, int64_t ldx, float* act_mean,
                                            awq_stream_t stream) {
  AWQ_TRY(check_matrix("X", X, N, K, ldx));
  if (K % 2 != 0) return fail(AWQ_ERR_INVALID_ARG, "K must be even");
  if (act_mean == nullptr) return fail(AWQ_ERR_INVALID_ARG, "act_mean is null");
  AWQ_TRY(check_act_chunks("X", N));
  const ActLayout l = act_layout(N, K);
  const uint64_t need = static_cast<uint64_t>(l.n_chunks) * static_cast<uint64_t>(K);
  if (need > AWQ_NOALLOC_SCRATCH_DOUBLES)
    return fail(AWQ_ERR_INVALID_ARG,
                "awq_act_stats_noalloc: ceil(N/256)*K = %llu fp64 partial sums exceed the fixed scratch of %llu "
                "(16 MiB); use awq_act_stats with a workspace",
                static_cast<unsigned long long>(need), static_cast<unsigned long long>(AWQ_NOALLOC_SCRATCH_DOUBLES));
  DeviceInfo* d = nullptr;
  AWQ_TRY(device_info(&d));
  double* part = nullptr;
  AWQ_TRY(act_scratch_address(&part));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // Each (chunk, column) entry the finaliser reads is written first by this call, so the scratch needs
  // no clearing; what the previous call left there is simply overwritten.
  AWQ_TRY(launch_act_stats(X, N, K, ldx, part, act_mean, d->sms, st));
  return ok();
}

namespace {
awq_status scale_fold(bool columns, const void* A, int64_t R, int64_t C, int64_t lda, const float* s, int op, void* out,
                      int64_t ldo, awq_stream_t stream) {
  AWQ_TRY(check_matrix("A", A, R, C, lda));
  AWQ_TRY(check_matrix("out", out, R, C, ldo));
  if (C % 8 != 0) return fail(AWQ_ERR_INVALID_ARG, "C (%lld) must be a multiple of 8", static_cast<long long>(C));
  if (s == nullptr || (columns && !aligned16(s))) return fail(AWQ_ERR_INVALID_ARG, "s is null or not 16-byte aligned");
  if (op != AWQ_SCALE_MULTIPLY && op != AWQ_SCALE_DIVIDE) return fail(AWQ_ERR_INVALID_ARG, "unknown op %d", op);
  if (A == out && lda != ldo) return fail(AWQ_ERR_INVALID_ARG, "in-place scaling needs lda == ldo");
  DeviceInfo* d = nullptr;
  AWQ_TRY(device_info(&d));
  const int64_t vecs = R * (C / 8);
  const int64_t blocks = std::min<int64_t>(static_cast<int64_t>(d->sms) * 16, (vecs + awq::kFoldThreads - 1) / awq::kFoldThreads);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (columns)
    awq::scale_fold_kernel<true><<<static_cast<unsigned>(blocks), awq::kFoldThreads, 0, st>>>(
        static_cast<const uint16_t*>(A), R, C, lda, s, op == AWQ_SCALE_DIVIDE, static_cast<uint16_t*>(out), ldo);
  else
    awq::scale_fold_kernel<false><<<static_cast<unsigned>(blocks), awq::kFoldThreads, 0, st>>>(
        static_cast<const uint16_t*>(A), R, C, lda, s, op == AWQ_SCALE_DIVIDE, static_cast<uint16_t*>(out), ldo);
  AWQ_TRY(check_launch("scale_fold_kernel"));
  return ok();
}
}  // namespace

extern "C" awq_status awq_scale_columns(const void* A, int64_t R, int64_t C, int64_t lda, const float* s, int op,
                                        void* out, int64_t ldo, awq_stream_t stream) {
  return scale_fold(true, A, R, C, lda, s, op, out, ldo, stream);
}

extern "C" awq_status awq_scale_rows(const void* A, int64_t R, int64_t C, int64_t lda, const float* s, int op,
                                     void* out, int64_t ldo, awq_stream_t stream) {
  return scale_fold(false, A, R, C, lda, s, op, out, ldo, stream);
}

namespace {
struct W4Layout {
  int64_t O_pad, G, n_rb;
  size_t steps_off, zeros_off, counter_off, xp_off, sx_off, partial_off, bytes;
};
constexpr int64_t kW4MaxRowBlocks = 65536;  // few-token counters reserved for O up to 8M rows
// [0, 512) status word and tile counter (cleared by each many-token call); [512, 512 + 256 KB) the
// few-token kernel's per-row-block counters, at the same place for every shape and written by nothing
// else, so they stay zero from one call to the next whatever the shapes; then the group-major steps and
// zeros (many tokens), and the few-token kernel's permuted copy of X' (64 rows), group sums and split-K
// partial sums.
W4Layout w4_layout(int64_t K, int64_t O) {
  W4Layout l;
  l.O_pad = (O + awq::lg::BN - 1) / awq::lg::BN * awq::lg::BN;
  l.G = K / 128;
  l.n_rb = (O + awq::dec::ROWS - 1) / awq::dec::ROWS;
  l.counter_off = 512;
  l.steps_off = l.counter_off + static_cast<size_t>(kW4MaxRowBlocks) * 4;
  l.zeros_off = align_up(l.steps_off + static_cast<size_t>(l.G) * l.O_pad * 4, 256);
  l.xp_off = align_up(l.zeros_off + static_cast<size_t>(l.G) * l.O_pad * 4, 256);
  l.sx_off = align_up(l.xp_off + static_cast<size_t>(awq::dec::MAX_NT) * K * 2, 256);
  l.partial_off = align_up(l.sx_off + static_cast<size_t>(l.G) * awq::dec::MAX_NT * 4, 256);
  const int64_t rb = std::min(l.n_rb, kW4MaxRowBlocks);
  l.bytes = align_up(l.partial_off + static_cast<size_t>(rb) * awq::dec::max_slices(rb) * awq::dec::MAX_NT *
                                         awq::dec::ROWS * 4,
                     256);
  return l;
}

// Few tokens: weight rows on the MMA's M side, groups split into slices until every SM has a share,
// slices added by the last CTA of each row block. One launch; the per-block counters are zero from the
// caller's initial zero fill and every call leaves them zero.
awq_status w4a16_decode(const void* X, int64_t M, int64_t K, int64_t ldx, const uint32_t* codes, const float* steps,
                        const float* zeros, int64_t O, void* Y, int64_t ldy, void* workspace, const W4Layout& l,
                        awq_stream_t stream) {
  DeviceInfo* d = nullptr;
  AWQ_TRY(device_info(&d));
  const int nt = static_cast<int>((M + 15) / 16 * 16);
  const int num_groups = static_cast<int>(K / 128);
  // one wave of CTAs; a slice holds an even number of groups (one code box covers two)
  // Slices sized for two CTAs per SM at 16 tokens and one above. (At the default shared-memory carveout a
  // cooperative launch of that many 16-token CTAs was refused as too large for one wave; preferring shared
  // memory in the carveout let them all fit, and the 16 x 28672 -> 8192 layer then ran slower, 74 against
  // 56 us.)
  int64_t slices = static_cast<int64_t>(nt <= 16 ? 2 : 1) * d->sms / l.n_rb;
  slices = std::max<int64_t>(1, std::min<int64_t>({slices, awq::dec::max_slices(l.n_rb), (num_groups + 1) / 2}));
  const int g_per = static_cast<int>(((num_groups + slices - 1) / slices + 1) / 2 * 2);
  slices = (num_groups + g_per - 1) / g_per;
  if (l.n_rb * slices >= (1ll << 31)) return fail(AWQ_ERR_INVALID_ARG, "O is too large");
  char* ws = static_cast<char*>(workspace);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint16_t* xp = reinterpret_cast<uint16_t*>(ws + l.xp_off);
  float* sx = reinterpret_cast<float*>(ws + l.sx_off);
  CUtensorMap tmX, tmC;
  AWQ_TRY(make_tmap(&tmX, xp, nt, K, K, nt));
  AWQ_TRY(make_tmap_codes_sw128(&tmC, codes, O, K / 8, awq::dec::ROWS));
  const int64_t ctas = l.n_rb * slices;
  awq::dec::decode_prep_kernel<<<static_cast<unsigned>(num_groups), awq::dec::PREP_THREADS, 0, st>>>(
      static_cast<const uint16_t*>(X), M, K, ldx, nt, xp, sx);
  AWQ_TRY(check_launch("decode_prep_kernel"));
  awq::dec::Params p;
  p.steps = steps;
  p.zeros = zeros;
  p.Y = static_cast<__nv_bfloat16*>(Y);
  p.partial = reinterpret_cast<float*>(ws + l.partial_off);
  p.counter = reinterpret_cast<unsigned int*>(ws + l.counter_off);
  p.sx = sx;
  p.M = M;
  p.O = O;
  p.G = l.G;
  p.ldy = ldy;
  p.num_groups = num_groups;
  p.g_per = g_per;
  p.slices = static_cast<int>(slices);
  p.idesc = awq::idesc_bf16_f32(awq::dec::ROWS, static_cast<uint32_t>(nt));
  p.status = reinterpret_cast<awq::DeviceStatus*>(ws);
  p.limit_ns = g_wait_limit_ns.load();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas));
  cfg.blockDim = dim3(awq::dec::THREADS);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];  // a programmatic dependent of the prep kernel: its prologue and first code
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // loads overlap it
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (nt == 16) {
    cfg.dynamicSmemBytes = awq::dec::Shape<16>::SMEM;
    AWQ_CUDA(cudaLaunchKernelEx(&cfg, awq::dec::w4a16_decode_kernel<16>, tmX, tmC, p));
  } else if (nt == 32) {
    cfg.dynamicSmemBytes = awq::dec::Shape<32>::SMEM;
    AWQ_CUDA(cudaLaunchKernelEx(&cfg, awq::dec::w4a16_decode_kernel<32>, tmX, tmC, p));
  } else if (nt == 48) {
    cfg.dynamicSmemBytes = awq::dec::Shape<48>::SMEM;
    AWQ_CUDA(cudaLaunchKernelEx(&cfg, awq::dec::w4a16_decode_kernel<48>, tmX, tmC, p));
  } else {
    cfg.dynamicSmemBytes = awq::dec::Shape<64>::SMEM;
    AWQ_CUDA(cudaLaunchKernelEx(&cfg, awq::dec::w4a16_decode_kernel<64>, tmX, tmC, p));
  }
  AWQ_TRY(check_launch("w4a16_decode_kernel"));
  return ok();
}
}  // namespace

extern "C" size_t awq_w4a16_workspace_size(int64_t K, int64_t O) {
  if (K < 128 || O < 1) return 0;
  return w4_layout(K, O).bytes;
}

extern "C" awq_status awq_w4a16_gemm(const void* X, int64_t M, int64_t K, int64_t ldx, const uint32_t* codes,
                                     const float* steps, const float* zeros, int64_t O, void* Y, int64_t ldy,
                                     void* workspace, size_t ws_bytes, awq_stream_t stream) {
  AWQ_TRY(check_matrix("X", X, M, K, ldx));
  AWQ_TRY(check_matrix("Y", Y, M, O, ldy));
  if (K % 128 != 0) return fail(AWQ_ERR_INVALID_ARG, "K (%lld) must be a multiple of 128", static_cast<long long>(K));
  if (O % 8 != 0) return fail(AWQ_ERR_INVALID_ARG, "O (%lld) must be a multiple of 8", static_cast<long long>(O));
  if (codes == nullptr || steps == nullptr || zeros == nullptr || !aligned16(codes))
    return fail(AWQ_ERR_INVALID_ARG, "codes (16-byte aligned), steps and zeros must be given");
  const W4Layout l = w4_layout(K, O);
  if (workspace == nullptr || ws_bytes < l.bytes)
    return fail(AWQ_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", l.bytes, workspace ? ws_bytes : 0);
  if (!aligned16(workspace)) return fail(AWQ_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
  if (M <= awq::dec::MAX_NT && l.n_rb <= kW4MaxRowBlocks)
    return w4a16_decode(X, M, K, ldx, codes, steps, zeros, O, Y, ldy, workspace, l, stream);
  const int64_t n_tiles_m = (M + awq::dq::TM - 1) / awq::dq::TM;
  const int64_t n_bands = l.O_pad / awq::dq::BN;
  if (n_tiles_m * n_bands >= (1ll << 31)) return fail(AWQ_ERR_INVALID_ARG, "too many tiles");
  DeviceInfo* d = nullptr;
  AWQ_TRY(device_info(&d));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  float* steps_t = reinterpret_cast<float*>(ws + l.steps_off);
  float* zeros_t = reinterpret_cast<float*>(ws + l.zeros_off);
  CUtensorMap tmX, tmC, tmS, tmZ, tmY;
  AWQ_TRY(make_tmap(&tmX, X, M, K, ldx, awq::lg::HALF));
  AWQ_TRY(make_tmap_plain(&tmY, Y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, M, O, ldy, awq::dq::Y_CHUNK, 32));
  AWQ_TRY(make_tmap_plain(&tmC, codes, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, O, K / 8, K / 8, awq::lg::BK / 8,
                          awq::lg::HALF));
  AWQ_TRY(make_tmap_plain(&tmS, steps_t, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, l.G, l.O_pad, l.O_pad, awq::lg::HALF, 1));
  AWQ_TRY(make_tmap_plain(&tmZ, zeros_t, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, l.G, l.O_pad, l.O_pad, awq::lg::HALF, 1));
  AWQ_CUDA(cudaMemsetAsync(ws, 0, 512, st));
  awq::dq::transpose_groups_kernel<<<dim3(static_cast<unsigned>(l.O_pad / 256), static_cast<unsigned>(l.G)), 256, 0,
                                     st>>>(steps, zeros, O, l.O_pad, l.G, steps_t, zeros_t);
  AWQ_TRY(check_launch("transpose_groups_kernel"));
  awq::dq::Params p;
  p.Y = static_cast<__nv_bfloat16*>(Y);
  p.M = M;
  p.O = O;
  p.K = K;
  p.ldy = ldy;
  p.n_tiles_m = static_cast<int>(n_tiles_m);
  p.n_bands = static_cast<int>(n_bands);
  p.num_kb = static_cast<int>(K / awq::lg::BK);
  p.num_tiles = static_cast<int>(n_tiles_m * n_bands);
  p.tile_counter = reinterpret_cast<unsigned int*>(ws + 20);
  p.status = reinterpret_cast<awq::DeviceStatus*>(ws);
  p.limit_ns = g_wait_limit_ns.load();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * d->w4_clusters));
  cfg.blockDim = dim3(awq::dq::THREADS);
  cfg.dynamicSmemBytes = awq::dq::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  AWQ_CUDA(cudaLaunchKernelEx(&cfg, awq::dq::w4a16_gemm_kernel, tmX, tmC, tmS, tmZ, tmY, p));
  AWQ_TRY(check_launch("w4a16_gemm_kernel"));
  return ok();
}
