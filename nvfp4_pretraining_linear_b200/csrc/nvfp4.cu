// C ABI of the NVFP4 linear-layer library (declared in include/nvfp4.h).
//
// Host side only: argument validation, tensor-map construction for the GEMM's
// TMA loads, and kernel launches on the caller's stream.  One translation unit
// holds every kernel (quantize.cuh, gemm.cuh, ns.cuh, lowrank.cuh) so that the
// module-scope device error word is shared by all of them.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdarg>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "nvfp4.h"
#include "common.cuh"
#include "gemm.cuh"
#include "lowrank.cuh"
#include "ns.cuh"
#include "quantize.cuh"
#include "selfcheck.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kWorkspaceBytes = 256;

thread_local char g_last_error[512] = "";

nvfp4_status fail(nvfp4_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

nvfp4_status cuda_fail(cudaError_t e, const char* what) {
  return fail(NVFP4_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

struct DeviceInfo {
  int sm_count = 0;
  bool gemm_attr = false;
  int pair_clusters = 0;    // co-resident CTA pairs of the pair GEMM kernel
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;

nvfp4_status device_info(DeviceInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(NVFP4_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceInfo& d = g_dev[dev];
  if (d.sm_count == 0) {
    e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  }
  if (!d.gemm_attr) {
    e = cudaFuncSetAttribute(nvfp4::gemm::gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             nvfp4::gemm::SMEM_BYTES);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemm)");
    using namespace nvfp4::gemm;
    for (auto kernel : {gemm_kernel_pair<EPI_BF16, 1, false>, gemm_kernel_pair<EPI_BF16_ACC, 1, false>,
                        gemm_kernel_pair<EPI_F32, 1, false>, gemm_kernel_pair<EPI_F32_ACC, 1, false>,
                        gemm_kernel_pair<EPI_BF16, 1, true>}) {
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM_BYTES);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemm pair)");
    }
    for (auto kernel : {gemm_kernel_pair<EPI_BF16, kMaxGroup, false>, gemm_kernel_pair<EPI_F32, kMaxGroup, false>}) {
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM_BYTES);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(grouped gemm pair)");
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * (d.sm_count / 2), 1, 1);
    cfg.blockDim = dim3(nvfp4::gemm::P_NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = nvfp4::gemm::P_SMEM_BYTES;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, gemm_kernel_pair<EPI_BF16, 1, false>, &cfg);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveClusters");
    d.pair_clusters = clusters;
    d.gemm_attr = true;
  }
  *out = &d;
  return NVFP4_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

nvfp4_status get_encoder(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  std::call_once(g_encode_once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  if (!g_encode) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  *fn = g_encode;
  return NVFP4_OK;
}

// Tensor map of packed E2M1 codes [rows][cols/2 bytes]: box of box_rows x box_bytes
// bytes, swizzled with box_bytes (128 or 64): the tensor cores' K-major operand layout.
nvfp4_status make_code_map(CUtensorMap* map, const nvfp4_tensor* t, uint32_t box_rows, uint32_t box_bytes) {
  PFN_cuTensorMapEncodeTiled_v12000 encode;
  nvfp4_status st = get_encoder(&encode);
  if (st != NVFP4_OK) return st;
  const cuuint64_t dims[2] = {(cuuint64_t)(t->cols / 2), (cuuint64_t)t->rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(t->cols / 2)};
  const cuuint32_t box[2] = {box_bytes, box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, t->codes, dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE,
                      box_bytes == 128u ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return NVFP4_OK;
}

// Tensor map of the output C [M x N] (row stride ldc elements) for the pair GEMM's
// epilogue stores: boxes of 32 rows x 128 bytes (64 BF16 or 32 FP32 columns),
// 128-byte swizzle.
nvfp4_status make_out_map(CUtensorMap* map, void* C, int64_t M, int64_t N, int64_t ldc, bool f32) {
  PFN_cuTensorMapEncodeTiled_v12000 encode;
  nvfp4_status st = get_encoder(&encode);
  if (st != NVFP4_OK) return st;
  const cuuint64_t esz = f32 ? 4u : 2u;
  const cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
  const cuuint64_t strides[1] = {(cuuint64_t)ldc * esz};
  const cuuint32_t box[2] = {(cuuint32_t)(128u / esz), 32u};
  const cuuint32_t estr[2] = {1u, 1u};
  CUresult r = encode(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, C, dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled(C) failed (%d)", (int)r);
  return NVFP4_OK;
}

// Tensor map over the tensor-core scale layout viewed as rows of 512-byte atoms (128 x
// 32-bit words): box of box_atoms atoms = one 128-row block x 64 * box_atoms K.
nvfp4_status make_scale_map(CUtensorMap* map, const nvfp4_tensor* t, uint32_t box_atoms) {
  PFN_cuTensorMapEncodeTiled_v12000 encode;
  nvfp4_status st = get_encoder(&encode);
  if (st != NVFP4_OK) return st;
  const int64_t atoms = ceil_div(t->rows, 128) * ceil_div(t->cols / 16, 4);
  const cuuint64_t dims[2] = {128u, (cuuint64_t)atoms};
  const cuuint64_t strides[1] = {512u};
  const cuuint32_t box[2] = {128u, box_atoms};
  const cuuint32_t estr[2] = {1u, 1u};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, t->scales, dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled(scales) failed (%d)", (int)r);
  return NVFP4_OK;
}

nvfp4_status check_tensor(const nvfp4_tensor* t, const char* name) {
  if (!t) return fail(NVFP4_ERR_INVALID_ARG, "%s is NULL", name);
  if (t->rows < 0 || t->cols < 0) return fail(NVFP4_ERR_INVALID_ARG, "%s has a negative extent", name);
  const bool empty = t->rows == 0 || t->cols == 0;   // an empty tensor needs only its tensor scale
  if (!t->tensor_scale || (!empty && (!t->codes || !t->scales)))
    return fail(NVFP4_ERR_INVALID_ARG, "%s has a NULL buffer", name);
  if (t->scale_layout != NVFP4_SCALE_ROWMAJOR && t->scale_layout != NVFP4_SCALE_MMA)
    return fail(NVFP4_ERR_INVALID_ARG, "%s.scale_layout is %d", name, t->scale_layout);
  if (t->reserved != 0) return fail(NVFP4_ERR_INVALID_ARG, "%s.reserved must be 0", name);
  if (t->cols % 16) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "%s.cols %lld is not a multiple of 16", name, (long long)t->cols);
  if (!aligned16(t->codes)) return fail(NVFP4_ERR_MISALIGNED, "%s.codes is not 16-byte aligned", name);
  return NVFP4_OK;
}

nvfp4::QuantLayout layout_of(const nvfp4_tensor* t) {
  nvfp4::QuantLayout L{};
  if (!t) return L;
  L.codes = t->codes;
  L.scales = t->scales;
  L.tensor_scale = t->tensor_scale;
  L.kgroups = ceil_div(t->cols / 16, 4);
  L.mma_layout = t->scale_layout == NVFP4_SCALE_MMA;
  return L;
}

// Each kernel instantiation needs its large dynamic shared memory opted in once
// per device; `done` must be a distinct object per instantiation.
template <typename Kernel>
cudaError_t ensure_smem(Kernel kernel, int bytes, bool (&done)[kMaxDevices], std::mutex& m) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(m);
  if (done[dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done[dev] = true;
  return e;
}

// Host-side fault injection for failure-detection tests: with NVFP4_INJECT_SKIP_TILE=n
// in the environment, the quantise pass never loads its tile n, so a compute warp's
// bounded wait expires and nvfp4_get_status reports NVFP4_ERR_TIMEOUT.  Nothing
// faults, traps or hangs; unset (the default) it costs one getenv per call.
int64_t injected_skip_tile() {
  const char* v = std::getenv("NVFP4_INJECT_SKIP_TILE");
  if (!v || !*v) return -1;
  char* end = nullptr;
  const long long n = std::strtoll(v, &end, 10);
  return (end && *end == '\0' && n >= 0) ? (int64_t)n : -1;
}

// The same for the pair GEMM: with NVFP4_INJECT_GEMM_SKIP_STAGE=n, CTA pair 0 never
// loads its K-stage number n, so the MMA issuers' bounded wait expires.
int64_t injected_gemm_skip_stage() {
  const char* v = std::getenv("NVFP4_INJECT_GEMM_SKIP_STAGE");
  if (!v || !*v) return -1;
  char* end = nullptr;
  const long long n = std::strtoll(v, &end, 10);
  return (end && *end == '\0' && n >= 0) ? (int64_t)n : -1;
}

// A quantise pass that directly follows its own amax pass in the stream is launched
// as a programmatic dependent of it (after_amax): it loads its first tiles while the
// amax pass finishes and waits for it before reading the maxima.
template <bool AM, bool ER, bool EC, bool SR, bool RR, bool RC, bool TD>
cudaError_t launch_tiles(const CUtensorMap& map, const nvfp4::QuantParams& p, int grid, cudaStream_t s,
                         bool after_amax = false) {
  static bool done[kMaxDevices] = {};
  static std::mutex m;
  auto kernel = nvfp4::quant_tile_kernel<AM, ER, EC, SR, RR, RC, TD>;
  cudaError_t e = ensure_smem(kernel, nvfp4::kQSmemBytes, done, m);
  if (e != cudaSuccess) return e;
  if (!after_amax) {
    kernel<<<grid, nvfp4::kQThreads, nvfp4::kQSmemBytes, s>>>(map, p);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(nvfp4::kQThreads);
  cfg.dynamicSmemBytes = nvfp4::kQSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, map, p);
}

template <bool ER, bool EC, bool SR, bool RR, bool RC>
cudaError_t dispatch_td(bool td, const CUtensorMap& m, const nvfp4::QuantParams& p, int g, cudaStream_t s, bool dep) {
  if constexpr (!SR && !RR && !RC) {
    if (td) return launch_tiles<false, ER, EC, false, false, false, true>(m, p, g, s, dep);
  }
  return launch_tiles<false, ER, EC, SR, RR, RC, false>(m, p, g, s, dep);
}

template <bool ER, bool EC, bool SR, bool RR>
cudaError_t dispatch_rc(bool rc, bool td, const CUtensorMap& m, const nvfp4::QuantParams& p, int g, cudaStream_t s,
                        bool dep) {
  if (rc) return dispatch_td<ER, EC, SR, RR, true>(td, m, p, g, s, dep);
  return dispatch_td<ER, EC, SR, RR, false>(td, m, p, g, s, dep);
}

template <bool ER, bool EC, bool SR>
cudaError_t dispatch_rr(bool rr, bool rc, bool td, const CUtensorMap& m, const nvfp4::QuantParams& p, int g,
                        cudaStream_t s, bool dep) {
  if (rr) return dispatch_rc<ER, EC, SR, true>(rc, td, m, p, g, s, dep);
  return dispatch_rc<ER, EC, SR, false>(rc, td, m, p, g, s, dep);
}

template <bool ER, bool EC>
cudaError_t dispatch_sr(bool sr, bool rr, bool rc, bool td, const CUtensorMap& m, const nvfp4::QuantParams& p, int g,
                        cudaStream_t s, bool dep) {
  if (sr) return dispatch_rr<ER, EC, true>(rr, rc, td, m, p, g, s, dep);
  return dispatch_rr<ER, EC, false>(rr, rc, td, m, p, g, s, dep);
}

// dep: the quantise pass follows its own amax pass in the stream (see launch_tiles).
cudaError_t dispatch_quant(bool er, bool ec, bool sr, bool rr, bool rc, bool td, const CUtensorMap& m,
                           const nvfp4::QuantParams& p, int g, cudaStream_t s, bool dep) {
  if (er && ec) return dispatch_sr<true, true>(sr, rr, rc, td, m, p, g, s, dep);
  if (er) return dispatch_sr<true, false>(sr, rr, rc, td, m, p, g, s, dep);
  return dispatch_sr<false, true>(sr, rr, rc, td, m, p, g, s, dep);
}

cudaError_t dispatch_amax(bool rr, bool rc, const CUtensorMap& m, const nvfp4::QuantParams& p, int g, cudaStream_t s) {
  if (rr && rc) return launch_tiles<true, false, false, false, true, true, false>(m, p, g, s);
  if (rc) return launch_tiles<true, false, false, false, false, true, false>(m, p, g, s);
  if (rr) return launch_tiles<true, false, false, false, true, false, false>(m, p, g, s);
  return launch_tiles<true, false, false, false, false, false, false>(m, p, g, s);
}

// Tensor map of a BF16 matrix [rows][cols] with row stride ld elements: 128 x 128 tiles,
// no swizzle, zero fill outside the matrix.
nvfp4_status make_input_map(CUtensorMap* map, const void* x, int64_t rows, int64_t cols, int64_t ld) {
  PFN_cuTensorMapEncodeTiled_v12000 encode;
  nvfp4_status st = get_encoder(&encode);
  if (st != NVFP4_OK) return st;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  const cuuint32_t box[2] = {(cuuint32_t)nvfp4::kTileCols, (cuuint32_t)nvfp4::kTileRows};
  const cuuint32_t estr[2] = {1u, 1u};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled(input) failed (%d)", (int)r);
  return NVFP4_OK;
}

// ------------------------------------------------------------------ fixed scratch
//
// Scratch for nvfp4_quantize_noalloc: the quantiser's amax accumulators live in
// this module-scope device array instead of a caller workspace.  Every GPU that
// loads the library holds these bytes until the process exits.  In host code
// the name is only a stand-in for the symbol: its device address is fetched
// with cudaGetSymbolAddress once per device and cached.
constexpr size_t kNoAllocScratchBytes = 256;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void* g_noalloc_addr[kMaxDevices] = {};
std::mutex g_noalloc_mutex;

nvfp4_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(NVFP4_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_addr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
    g_noalloc_addr[dev] = ptr;
  }
  *out = g_noalloc_addr[dev];
  return NVFP4_OK;
}

}  // namespace

extern "C" {

int nvfp4_version(void) { return 200; }

size_t nvfp4_workspace_size(void) { return kWorkspaceBytes; }

size_t nvfp4_scales_bytes(int64_t rows, int64_t cols, int32_t scale_layout) {
  if (rows < 0 || cols < 0) return 0;
  if (scale_layout == NVFP4_SCALE_MMA) return (size_t)(ceil_div(rows, 128) * 128) * (size_t)(ceil_div(cols / 16, 4) * 4);
  return (size_t)rows * (size_t)(cols / 16);
}

const char* nvfp4_last_error_string(void) { return g_last_error; }

nvfp4_status nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld, const nvfp4_quant_opts* opts,
                            nvfp4_tensor* out_row, nvfp4_tensor* out_col, void* workspace, size_t workspace_bytes,
                            void* stream) {
  if (!opts) return fail(NVFP4_ERR_INVALID_ARG, "opts is NULL");
  if (!out_row && !out_col) return fail(NVFP4_ERR_INVALID_ARG, "no output layout requested");
  if (rows < 0 || cols < 0) return fail(NVFP4_ERR_INVALID_ARG, "negative extent");
  if (cols % 16) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "cols %lld is not a multiple of 16", (long long)cols);
  if ((out_col || opts->block_2d) && rows % 16)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "rows %lld is not a multiple of 16 (col layout / 2D blocks)", (long long)rows);
  if (rows > 0 && cols > 0) {
    if (!x) return fail(NVFP4_ERR_INVALID_ARG, "x is NULL");
    if (ld < cols) return fail(NVFP4_ERR_INVALID_ARG, "ld %lld < cols %lld", (long long)ld, (long long)cols);
    if (!aligned16(x) || ld % 8) return fail(NVFP4_ERR_MISALIGNED, "x rows are not 16-byte aligned");
  }
  if (opts->reserved) return fail(NVFP4_ERR_INVALID_ARG, "opts.reserved must be 0");
  if (opts->block_2d && (opts->stochastic || opts->rht_row || opts->rht_col))
    return fail(NVFP4_ERR_INVALID_ARG, "2D weight blocks exclude stochastic rounding and the RHT");
  if (opts->offset >> 32) return fail(NVFP4_ERR_INVALID_ARG, "opts.offset must be < 2^32");
  if (opts->rht_signs >> 16) return fail(NVFP4_ERR_INVALID_ARG, "opts.rht_signs has bits above 15");
  if (opts->rht_row && !out_row) return fail(NVFP4_ERR_INVALID_ARG, "rht_row without a row layout");
  if (opts->rht_col && !out_col) return fail(NVFP4_ERR_INVALID_ARG, "rht_col without a col layout");
  nvfp4_status st;
  if (out_row) {
    if ((st = check_tensor(out_row, "out_row")) != NVFP4_OK) return st;
    if (out_row->rows != rows || out_row->cols != cols)
      return fail(NVFP4_ERR_INVALID_ARG, "out_row is %lldx%lld, x is %lldx%lld", (long long)out_row->rows,
                  (long long)out_row->cols, (long long)rows, (long long)cols);
  }
  if (out_col) {
    if ((st = check_tensor(out_col, "out_col")) != NVFP4_OK) return st;
    if (out_col->rows != cols || out_col->cols != rows)
      return fail(NVFP4_ERR_INVALID_ARG, "out_col is %lldx%lld, expected %lldx%lld", (long long)out_col->rows,
                  (long long)out_col->cols, (long long)cols, (long long)rows);
  }
  const float* amax = opts->amax_in;
  if (!amax) {
    if (!workspace || workspace_bytes < kWorkspaceBytes)
      return fail(NVFP4_ERR_WORKSPACE, "workspace of %zu bytes needed", kWorkspaceBytes);
    if (!aligned16(workspace)) return fail(NVFP4_ERR_MISALIGNED, "workspace is not 16-byte aligned");
  }
  DeviceInfo* dev;
  if ((st = device_info(&dev)) != NVFP4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (rows == 0 || cols == 0) {
    // nothing to encode: S = 1 for every requested layout
    nvfp4::empty_tensor_scales_kernel<<<1, 32, 0, s>>>(out_row ? out_row->tensor_scale : nullptr,
                                                       out_col ? out_col->tensor_scale : nullptr, opts->amax_out);
    e = cudaGetLastError();
    return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "quantize launch");
  }
  CUtensorMap map;
  if ((st = make_input_map(&map, x, rows, cols, ld)) != NVFP4_OK) return st;
  nvfp4::QuantParams p{};
  p.rows = rows;
  p.cols = cols;
  p.tiles_c = ceil_div(cols, nvfp4::kTileCols);
  p.tiles = ceil_div(rows, nvfp4::kTileRows) * p.tiles_c;
  p.row = layout_of(out_row);
  p.col = layout_of(out_col);
  p.amax_out = opts->amax_out;
  // Philox round keys of the seed (the key schedule of Philox4x32-10, precomputed)
  for (int r = 0; r < 10; ++r) {
    p.rk[r] = (uint32_t)opts->seed + (uint32_t)r * 0x9E3779B9u;
    p.rk[10 + r] = (uint32_t)(opts->seed >> 32) + (uint32_t)r * 0xBB67AE85u;
  }
  p.offset = (uint32_t)opts->offset;
  p.signs = opts->rht_signs;
  p.skip_tile = -1;
  const int grid = (int)std::min<int64_t>(p.tiles, (int64_t)dev->sm_count * nvfp4::kQCtasPerSm);
  if (!amax) {
    unsigned* acc = static_cast<unsigned*>(workspace);
    e = cudaMemsetAsync(acc, 0, 3 * sizeof(unsigned), s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(workspace)");
    p.amax_acc = acc;
    e = dispatch_amax(opts->rht_row != 0, opts->rht_col != 0, map, p, grid, s);
    if (e != cudaSuccess) return cuda_fail(e, "amax launch");
    amax = reinterpret_cast<const float*>(acc);
  }
  p.amax = amax;
  p.amax_acc = nullptr;
  p.skip_tile = injected_skip_tile();
  e = dispatch_quant(out_row != nullptr, out_col != nullptr, opts->stochastic != 0, opts->rht_row != 0,
                     opts->rht_col != 0, opts->block_2d != 0, map, p, grid, s, opts->amax_in == nullptr);
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  return NVFP4_OK;
}

nvfp4_status nvfp4_dequantize(const nvfp4_tensor* q, void* out, int64_t ldo, int32_t out_dtype, void* stream) {
  nvfp4_status st = check_tensor(q, "q");
  if (st != NVFP4_OK) return st;
  if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_F32) return fail(NVFP4_ERR_INVALID_ARG, "out_dtype %d", out_dtype);
  const int64_t total = q->rows * (q->cols / 16);
  if (total == 0) return NVFP4_OK;
  if (!out) return fail(NVFP4_ERR_INVALID_ARG, "out is NULL");
  if (ldo < q->cols) return fail(NVFP4_ERR_INVALID_ARG, "ldo < cols");
  if (!aligned16(out) || (ldo * (out_dtype == NVFP4_OUT_F32 ? 4 : 2)) % 16)
    return fail(NVFP4_ERR_MISALIGNED, "out rows are not 16-byte aligned");
  DeviceInfo* dev;
  if ((st = device_info(&dev)) != NVFP4_OK) return st;
  const int grid = (int)std::min<int64_t>(ceil_div(total, 256), (int64_t)dev->sm_count * 16);
  nvfp4::dequantize_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      q->codes, q->scales, q->tensor_scale, q->rows, q->cols, q->scale_layout == NVFP4_SCALE_MMA,
      ceil_div(q->cols / 16, 4), out, ldo, out_dtype == NVFP4_OUT_F32);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "dequantize launch");
  return NVFP4_OK;
}

namespace {
// Low-rank operands of a GEMM that adds U V^T inside its accumulator (nvfp4_gemm_lowrank):
// U [M x rank], V [N x rank], BF16, row strides ldu, ldv elements.
struct LowRank {
  const void* U = nullptr;
  int64_t ldu = 0;
  const void* V = nullptr;
  int64_t ldv = 0;
  int32_t rank = 0;
};

// Tensor map of a BF16 low-rank factor [rows x rank] (row stride ld elements): boxes of
// 128 rows x 64 elements (128 bytes, zero-filled past the rank), 128-byte swizzle -- the
// K-major operand layout of the low-rank stage's BF16 MMAs.
nvfp4_status make_lowrank_map(CUtensorMap* map, const void* X, int64_t rows, int64_t ld, int32_t rank) {
  PFN_cuTensorMapEncodeTiled_v12000 encode;
  nvfp4_status st = get_encoder(&encode);
  if (st != NVFP4_OK) return st;
  const cuuint64_t dims[2] = {(cuuint64_t)rank, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 2u};
  const cuuint32_t box[2] = {64u, 128u};
  const cuuint32_t estr[2] = {1u, 1u};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(X), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled(low-rank factor) failed (%d)", (int)r);
  return NVFP4_OK;
}

// Tensor maps and the per-problem fields of one CTA-pair GEMM problem (p holds the shape,
// stage and scale fields filled by the caller): 256-element K-stages (128-byte code
// boxes, four scale tiles per stage), 256-row tiles; the output store map unless the
// epilogue accumulates in FP32 (which writes C directly).
nvfp4_status pair_problem(const nvfp4_tensor* A, const nvfp4_tensor* B, void* C, int64_t ldc, int32_t out_dtype,
                          int32_t accumulate, nvfp4::gemm::Params* p, nvfp4::gemm::PairMaps* maps) {
  nvfp4_status st;
  if ((st = make_code_map(&maps->a, A, 128, nvfp4::gemm::BK_BYTES)) != NVFP4_OK) return st;
  if ((st = make_code_map(&maps->b, B, 128, nvfp4::gemm::BK_BYTES)) != NVFP4_OK) return st;
  if ((st = make_scale_map(&maps->sfa, A, nvfp4::gemm::BK / nvfp4::gemm::MMA_K)) != NVFP4_OK) return st;
  if ((st = make_scale_map(&maps->sfb, B, nvfp4::gemm::BK / nvfp4::gemm::MMA_K)) != NVFP4_OK) return st;
  const bool f32 = out_dtype == NVFP4_OUT_F32;
  if (!(f32 && accumulate) && (st = make_out_map(&maps->c, C, A->rows, B->rows, ldc, f32)) != NVFP4_OK) return st;
  p->num_m = (int32_t)ceil_div(A->rows, nvfp4::gemm::P_BM);
  p->group_m = 16;
  return NVFP4_OK;
}

// Launch configuration of the pair kernel: clusters of 2 CTAs, one pair per two SMs up to
// the co-resident maximum, never more pairs than tiles.  It is a programmatic dependent
// of the kernel before it in the stream (attr[1]): its set-up overlaps that kernel's
// last CTAs, and it waits for that kernel before touching global memory.
void pair_launch_config(cudaLaunchConfig_t* cfg, cudaLaunchAttribute (&attr)[2], int64_t tiles, int pair_clusters,
                        cudaStream_t s) {
  std::memset(cfg, 0, sizeof(*cfg));
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  const int pairs = (int)std::min<int64_t>(tiles, pair_clusters);
  cfg->gridDim = dim3(2 * pairs, 1, 1);
  cfg->blockDim = dim3(nvfp4::gemm::P_NUM_THREADS, 1, 1);
  cfg->dynamicSmemBytes = nvfp4::gemm::P_SMEM_BYTES;
  cfg->stream = s;
  cfg->attrs = attr;
  cfg->numAttrs = 2;
}

// nvfp4_gemm; with amax_out (3 floats) the maxima of nvfp4_gemm_amax; with a low-rank
// pair the U V^T term of nvfp4_gemm_lowrank.
nvfp4_status gemm_impl(const nvfp4_tensor* A, const nvfp4_tensor* B, void* C, int64_t ldc, int32_t out_dtype,
                       float alpha, int32_t accumulate, float* amax_out, uint32_t rht_signs, void* stream,
                       const LowRank* lr = nullptr) {
  nvfp4_status st;
  if ((st = check_tensor(A, "A")) != NVFP4_OK) return st;
  if ((st = check_tensor(B, "B")) != NVFP4_OK) return st;
  if (A->cols != B->cols) return fail(NVFP4_ERR_INVALID_ARG, "A.cols %lld != B.cols %lld", (long long)A->cols, (long long)B->cols);
  if (A->scale_layout != NVFP4_SCALE_MMA || B->scale_layout != NVFP4_SCALE_MMA)
    return fail(NVFP4_ERR_INVALID_ARG, "GEMM operands need the tensor-core scale layout");
  if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_F32) return fail(NVFP4_ERR_INVALID_ARG, "out_dtype %d", out_dtype);
  const int64_t M = A->rows, N = B->rows, K = A->cols;
  if (M % 128 || N % 128 || K % 64)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "GEMM needs M %% 128, N %% 128, K %% 64 == 0 (got %lld, %lld, %lld)",
                (long long)M, (long long)N, (long long)K);
  if (M > (1ll << 31) - 128 || N > (1ll << 31) - 256 || K > (1ll << 31) - 256)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "GEMM extent above 2^31");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (amax_out) {
    if (out_dtype != NVFP4_OUT_BF16 || accumulate)
      return fail(NVFP4_ERR_INVALID_ARG, "the output maxima need BF16 output without accumulation");
    if (M != 0 && M < 256) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "the output maxima need M >= 256");
    const cudaError_t e = cudaMemsetAsync(amax_out, 0, 3 * sizeof(float), s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(amax_out)");
  }
  if (M == 0 || N == 0) return NVFP4_OK;
  if (!C) return fail(NVFP4_ERR_INVALID_ARG, "C is NULL");
  if (ldc < N) return fail(NVFP4_ERR_INVALID_ARG, "ldc < N");
  if (!aligned16(C) || (ldc * (out_dtype == NVFP4_OUT_F32 ? 4 : 2)) % 16)
    return fail(NVFP4_ERR_MISALIGNED, "C rows are not 16-byte aligned");
  if (!aligned16(A->scales) || !aligned16(B->scales)) return fail(NVFP4_ERR_MISALIGNED, "scales not 16-byte aligned");
  if (K == 0) {
    // empty contraction: C = 0 (or unchanged when accumulating)
    if (accumulate) return NVFP4_OK;
    const size_t esz = out_dtype == NVFP4_OUT_F32 ? 4 : 2;
    cudaError_t e = cudaMemset2DAsync(C, (size_t)ldc * esz, 0, (size_t)N * esz, (size_t)M, s);
    return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "cudaMemset2DAsync");
  }
  DeviceInfo* dev;
  if ((st = device_info(&dev)) != NVFP4_OK) return st;
  nvfp4::gemm::Params p{};
  p.M = (int32_t)M;
  p.N = (int32_t)N;
  p.K = (int32_t)K;
  p.num_n = (int32_t)ceil_div(N, nvfp4::gemm::BN);
  p.num_k_stages = (int32_t)ceil_div(K, nvfp4::gemm::BK);
  const int64_t tail = K % nvfp4::gemm::BK;
  p.tail_atoms = tail ? (int32_t)(tail / nvfp4::gemm::MMA_K) : nvfp4::gemm::BK / nvfp4::gemm::MMA_K;
  p.sfa = A->scales;
  p.sfb = B->scales;
  p.sf_kgroups = K / 64;
  p.sf_kgroups_a = K / 64;
  p.scale_a = A->tensor_scale;
  p.scale_b = B->tensor_scale;
  p.alpha = alpha;
  p.C = C;
  p.ldc = ldc;
  p.out_f32 = out_dtype == NVFP4_OUT_F32;
  p.accumulate = accumulate != 0;
  p.amax_acc = reinterpret_cast<unsigned*>(amax_out);
  p.rht_signs = rht_signs & 0xFFFFu;
  p.skip_stage = injected_gemm_skip_stage();
  cudaError_t e;
  if (amax_out && dev->pair_clusters == 0)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "the output maxima need the CTA-pair GEMM, not available on this device");
  if (lr && (M < 256 || dev->pair_clusters == 0))
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "the low-rank term needs M >= 256 and the CTA-pair GEMM");
  p.lr_ksteps = lr ? lr->rank / 16 : 0;
  // CTA pairs unless M = 128 leaves more 256-column tiles than pairs: a 128-row problem
  // runs on the pair kernel with half of each pair tile empty, which is faster only
  // while every tile gets a pair of SMs (one wave); past that the single-CTA kernel's
  // 128 x 256 tiles fill the SMs in fewer waves.
  const bool use_pair = dev->pair_clusters > 0 &&
                        (M >= 256 || amax_out || ceil_div(N, nvfp4::gemm::BN) <= (int64_t)dev->pair_clusters);
  if (use_pair) {
    // CTA pairs, 256 x 256 tiles: a table of one problem
    nvfp4::gemm::PairGroup<1> grp;
    std::memset(&grp, 0, sizeof(grp));
    if ((st = pair_problem(A, B, C, ldc, out_dtype, accumulate, &p, &grp.maps[0])) != NVFP4_OK) return st;
    if (lr) {
      if ((st = make_lowrank_map(&grp.u, lr->U, M, lr->ldu, lr->rank)) != NVFP4_OK) return st;
      if ((st = make_lowrank_map(&grp.v, lr->V, N, lr->ldv, lr->rank)) != NVFP4_OK) return st;
    }
    grp.p[0] = p;
    grp.tile_end[0] = p.num_m * p.num_n;
    grp.count = 1;
    using namespace nvfp4::gemm;
    const bool f32 = out_dtype == NVFP4_OUT_F32;
    // the low-rank stage is only taken with a plain BF16 output (nvfp4_gemm_lowrank)
    auto kernel = lr ? gemm_kernel_pair<EPI_BF16, 1, true>
                  : f32 ? (accumulate ? gemm_kernel_pair<EPI_F32_ACC, 1, false> : gemm_kernel_pair<EPI_F32, 1, false>)
                        : (accumulate ? gemm_kernel_pair<EPI_BF16_ACC, 1, false> : gemm_kernel_pair<EPI_BF16, 1, false>);
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[2];
    pair_launch_config(&cfg, attr, grp.tile_end[0], dev->pair_clusters, s);
    e = cudaLaunchKernelEx(&cfg, kernel, grp);
  } else {
    CUtensorMap map_a, map_b;
    if ((st = make_code_map(&map_a, A, nvfp4::gemm::BM, nvfp4::gemm::BK_BYTES)) != NVFP4_OK) return st;
    if ((st = make_code_map(&map_b, B, nvfp4::gemm::BN, nvfp4::gemm::BK_BYTES)) != NVFP4_OK) return st;
    p.num_m = (int32_t)(M / nvfp4::gemm::BM);
    p.group_m = 16;
    const int64_t tiles = (int64_t)p.num_m * p.num_n;
    const int grid = (int)std::min<int64_t>(tiles, dev->sm_count);
    nvfp4::gemm::gemm_kernel<<<grid, nvfp4::gemm::NUM_THREADS, nvfp4::gemm::SMEM_BYTES, s>>>(map_a, map_b, p);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
  return NVFP4_OK;
}
}  // namespace

nvfp4_status nvfp4_gemm(const nvfp4_tensor* A, const nvfp4_tensor* B, void* C, int64_t ldc, int32_t out_dtype,
                        float alpha, int32_t accumulate, void* stream) {
  return gemm_impl(A, B, C, ldc, out_dtype, alpha, accumulate, nullptr, 0u, stream);
}

nvfp4_status nvfp4_gemm_amax(const nvfp4_tensor* A, const nvfp4_tensor* B, void* C, int64_t ldc, float alpha,
                             uint32_t rht_signs, float* amax_out, void* stream) {
  if (!amax_out) return fail(NVFP4_ERR_INVALID_ARG, "amax_out is NULL");
  if (reinterpret_cast<uintptr_t>(amax_out) % 4) return fail(NVFP4_ERR_MISALIGNED, "amax_out is not 4-byte aligned");
  return gemm_impl(A, B, C, ldc, NVFP4_OUT_BF16, alpha, 0, amax_out, rht_signs, stream);
}

nvfp4_status nvfp4_gemm_lowrank(const nvfp4_tensor* A, const nvfp4_tensor* B, const void* U, int64_t ldu,
                                const void* V, int64_t ldv, int32_t rank, void* C, int64_t ldc, void* stream) {
  if (rank != 16 && rank != 32 && rank != 48 && rank != 64)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "rank %d is not 16, 32, 48 or 64", rank);
  if (!U || !V) return fail(NVFP4_ERR_INVALID_ARG, "U or V is NULL");
  if (ldu < rank || ldv < rank) return fail(NVFP4_ERR_INVALID_ARG, "ldu or ldv < rank");
  if (!aligned16(U) || !aligned16(V) || ldu % 8 || ldv % 8)
    return fail(NVFP4_ERR_MISALIGNED, "U and V rows must be 16-byte aligned");
  LowRank lr;
  lr.U = U;
  lr.ldu = ldu;
  lr.V = V;
  lr.ldv = ldv;
  lr.rank = rank;
  return gemm_impl(A, B, C, ldc, NVFP4_OUT_BF16, 1.0f, 0, nullptr, 0u, stream, &lr);
}

nvfp4_status nvfp4_gemm_grouped(const nvfp4_tensor* const* A, const nvfp4_tensor* const* B, void* const* C,
                                const int64_t* ldc, int32_t count, int32_t out_dtype, void* stream) {
  if (!A || !B || !C || !ldc) return fail(NVFP4_ERR_INVALID_ARG, "NULL problem array");
  if (count < 1 || count > nvfp4::gemm::kMaxGroup)
    return fail(NVFP4_ERR_INVALID_ARG, "count %d outside 1 .. %d", count, nvfp4::gemm::kMaxGroup);
  if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_F32) return fail(NVFP4_ERR_INVALID_ARG, "out_dtype %d", out_dtype);
  nvfp4::gemm::PairGroup<nvfp4::gemm::kMaxGroup> grp;
  std::memset(&grp, 0, sizeof(grp));
  nvfp4_status st;
  for (int i = 0; i < count; ++i) {
    char an[16], bn[16];
    std::snprintf(an, sizeof(an), "A[%d]", i);
    std::snprintf(bn, sizeof(bn), "B[%d]", i);
    if ((st = check_tensor(A[i], an)) != NVFP4_OK) return st;
    if ((st = check_tensor(B[i], bn)) != NVFP4_OK) return st;
    if (A[i]->cols != B[i]->cols) return fail(NVFP4_ERR_INVALID_ARG, "problem %d: A.cols != B.cols", i);
    if (A[i]->scale_layout != NVFP4_SCALE_MMA || B[i]->scale_layout != NVFP4_SCALE_MMA)
      return fail(NVFP4_ERR_INVALID_ARG, "problem %d: GEMM operands need the tensor-core scale layout", i);
    const int64_t M = A[i]->rows, N = B[i]->rows, K = A[i]->cols;
    if (M <= 0 || N <= 0 || K <= 0 || M % 128 || N % 128 || K % 64)
      return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "problem %d: needs M, N, K > 0, M %% 128, N %% 128, K %% 64 == 0", i);
    if (M > (1ll << 31) - 128 || N > (1ll << 31) - 256 || K > (1ll << 31) - 256)
      return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "problem %d: extent above 2^31", i);
    if (!C[i]) return fail(NVFP4_ERR_INVALID_ARG, "C[%d] is NULL", i);
    if (ldc[i] < N) return fail(NVFP4_ERR_INVALID_ARG, "ldc[%d] < N", i);
    if (!aligned16(C[i]) || (ldc[i] * (out_dtype == NVFP4_OUT_F32 ? 4 : 2)) % 16)
      return fail(NVFP4_ERR_MISALIGNED, "C[%d] rows are not 16-byte aligned", i);
    if (!aligned16(A[i]->scales) || !aligned16(B[i]->scales))
      return fail(NVFP4_ERR_MISALIGNED, "problem %d: scales not 16-byte aligned", i);
  }
  DeviceInfo* dev;
  if ((st = device_info(&dev)) != NVFP4_OK) return st;
  if (dev->pair_clusters == 0) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "the grouped GEMM needs the CTA-pair kernel");
  int64_t tiles = 0;
  for (int i = 0; i < count; ++i) {
    nvfp4::gemm::Params& p = grp.p[i];
    const int64_t M = A[i]->rows, N = B[i]->rows, K = A[i]->cols;
    p.M = (int32_t)M;
    p.N = (int32_t)N;
    p.K = (int32_t)K;
    p.num_n = (int32_t)ceil_div(N, nvfp4::gemm::BN);
    p.num_k_stages = (int32_t)ceil_div(K, nvfp4::gemm::BK);
    const int64_t tail = K % nvfp4::gemm::BK;
    p.tail_atoms = tail ? (int32_t)(tail / nvfp4::gemm::MMA_K) : nvfp4::gemm::BK / nvfp4::gemm::MMA_K;
    p.sfa = A[i]->scales;
    p.sfb = B[i]->scales;
    p.sf_kgroups = K / 64;
    p.sf_kgroups_a = K / 64;
    p.scale_a = A[i]->tensor_scale;
    p.scale_b = B[i]->tensor_scale;
    p.alpha = 1.0f;
    p.C = C[i];
    p.ldc = ldc[i];
    p.out_f32 = out_dtype == NVFP4_OUT_F32;
    p.skip_stage = i == 0 ? injected_gemm_skip_stage() : -1;
    if ((st = pair_problem(A[i], B[i], C[i], ldc[i], out_dtype, 0, &p, &grp.maps[i])) != NVFP4_OK) return st;
    tiles += (int64_t)p.num_m * p.num_n;
    if (tiles > INT32_MAX) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "more than 2^31 tiles");
    grp.tile_end[i] = (int32_t)tiles;
  }
  grp.count = count;
  using namespace nvfp4::gemm;
  auto kernel = out_dtype == NVFP4_OUT_F32 ? gemm_kernel_pair<EPI_F32, kMaxGroup, false>
                                                 : gemm_kernel_pair<EPI_BF16, kMaxGroup, false>;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  pair_launch_config(&cfg, attr, tiles, dev->pair_clusters, static_cast<cudaStream_t>(stream));
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, grp);
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "grouped gemm launch");
}

nvfp4_status nvfp4_linear_fwd(const void* X, int64_t M, int64_t K, int64_t ldx, const nvfp4_tensor* Wq_row, void* Y,
                              int64_t ldy, int32_t out_dtype, nvfp4_tensor* Xq_row, nvfp4_tensor* Xq_col,
                              uint32_t rht_signs, void* workspace, size_t workspace_bytes, void* stream) {
  nvfp4_status st = check_tensor(Wq_row, "Wq_row");
  if (st != NVFP4_OK) return st;
  if (Wq_row->cols != K) return fail(NVFP4_ERR_INVALID_ARG, "Wq_row.cols %lld != K %lld", (long long)Wq_row->cols, (long long)K);
  if (!Xq_row) return fail(NVFP4_ERR_INVALID_ARG, "Xq_row is NULL");
  if (M % 128 || Wq_row->rows % 128 || K % 64) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "linear needs M %% 128, N %% 128, K %% 64 == 0");
  nvfp4_quant_opts o{};
  o.rht_col = Xq_col != nullptr;
  o.rht_signs = rht_signs;
  if ((st = nvfp4_quantize(X, M, K, ldx, &o, Xq_row, Xq_col, workspace, workspace_bytes, stream)) != NVFP4_OK) return st;
  return nvfp4_gemm(Xq_row, Wq_row, Y, ldy, out_dtype, 1.0f, 0, stream);
}

nvfp4_status nvfp4_linear_dgrad(const void* dY, int64_t M, int64_t N, int64_t ldy, const nvfp4_tensor* Wq_col,
                                void* dX, int64_t ldx, int32_t out_dtype, nvfp4_tensor* dYq_row, nvfp4_tensor* dYq_col,
                                uint64_t seed, uint64_t offset, uint32_t rht_signs, void* workspace,
                                size_t workspace_bytes, void* stream) {
  nvfp4_status st = check_tensor(Wq_col, "Wq_col");
  if (st != NVFP4_OK) return st;
  if (Wq_col->cols != N) return fail(NVFP4_ERR_INVALID_ARG, "Wq_col.cols %lld != N %lld", (long long)Wq_col->cols, (long long)N);
  if (!dYq_row) return fail(NVFP4_ERR_INVALID_ARG, "dYq_row is NULL");
  if (M % 128 || Wq_col->rows % 128 || N % 64) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "dgrad needs M %% 128, K %% 128, N %% 64 == 0");
  nvfp4_quant_opts o{};
  o.stochastic = 1;
  o.rht_col = dYq_col != nullptr;
  o.seed = seed;
  o.offset = offset;
  o.rht_signs = rht_signs;
  if ((st = nvfp4_quantize(dY, M, N, ldy, &o, dYq_row, dYq_col, workspace, workspace_bytes, stream)) != NVFP4_OK) return st;
  return nvfp4_gemm(dYq_row, Wq_col, dX, ldx, out_dtype, 1.0f, 0, stream);
}

nvfp4_status nvfp4_linear_wgrad(const nvfp4_tensor* dYq_col, const nvfp4_tensor* Xq_col, void* dW, int64_t ldw,
                                int32_t out_dtype, int32_t accumulate, void* stream) {
  return nvfp4_gemm(dYq_col, Xq_col, dW, ldw, out_dtype, 1.0f, accumulate, stream);
}

}  // extern "C"

namespace {

// Workspace of nvfp4_newton_schulz, each part 256-byte aligned: the quantiser's
// scratch, the scalars (FP64 sum of squares, three tensor scales), the NVFP4 row
// and col layouts of X [m x n], the BF16 residual R [m x m] and its row layout.
struct NsLayout {
  size_t quant_ws, scalars, xr_codes, xr_scales, xc_codes, xc_scales, r, rr_codes, rr_scales, total;
};

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

NsLayout ns_layout(int64_t m, int64_t n) {
  NsLayout L{};
  size_t o = 0;
  auto take = [&o](size_t bytes) {
    const size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  L.quant_ws = take(kWorkspaceBytes);
  L.scalars = take(64);
  L.xr_codes = take((size_t)m * (size_t)n / 2);
  L.xr_scales = take(nvfp4_scales_bytes(m, n, NVFP4_SCALE_MMA));
  L.xc_codes = take((size_t)n * (size_t)m / 2);
  L.xc_scales = take(nvfp4_scales_bytes(n, m, NVFP4_SCALE_MMA));
  L.r = take((size_t)m * (size_t)m * 2);
  L.rr_codes = take((size_t)m * (size_t)m / 2);
  L.rr_scales = take(nvfp4_scales_bytes(m, m, NVFP4_SCALE_MMA));
  L.total = o;
  return L;
}

bool ns_shape_ok(int64_t m, int64_t n) {
  return m > 0 && n > 0 && m % 128 == 0 && n % 128 == 0 && m < (1ll << 30) && n < (1ll << 30);
}

}  // namespace

extern "C" {

size_t nvfp4_newton_schulz_workspace_size(int64_t m, int64_t n) {
  return ns_shape_ok(m, n) ? ns_layout(m, n).total : 0;
}

nvfp4_status nvfp4_newton_schulz(const void* G, int64_t m, int64_t n, int64_t ldg, void* X, int64_t ldx, int32_t iters,
                                 int32_t normalize, float* norm_out, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  if (!ns_shape_ok(m, n))
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "Newton-Schulz needs m, n > 0 and multiples of 128 (got %lld, %lld)",
                (long long)m, (long long)n);
  if (!G || !X) return fail(NVFP4_ERR_INVALID_ARG, "G or X is NULL");
  if (iters < 0) return fail(NVFP4_ERR_INVALID_ARG, "iters %d < 0", iters);
  if (ldg < n || ldx < n) return fail(NVFP4_ERR_INVALID_ARG, "ldg or ldx < n");
  if (!aligned16(G) || !aligned16(X) || ldg % 8 || ldx % 8)
    return fail(NVFP4_ERR_MISALIGNED, "G and X rows must be 16-byte aligned");
  if (G == X && ldg != ldx) return fail(NVFP4_ERR_INVALID_ARG, "in-place use needs ldg == ldx");
  if (norm_out && reinterpret_cast<uintptr_t>(norm_out) % 4) return fail(NVFP4_ERR_MISALIGNED, "norm_out alignment");
  const NsLayout L = ns_layout(m, n);
  if (!workspace || workspace_bytes < L.total)
    return fail(NVFP4_ERR_WORKSPACE, "Newton-Schulz needs %zu bytes of workspace", L.total);
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(NVFP4_ERR_MISALIGNED, "workspace is not 256-byte aligned");
  DeviceInfo* dev;
  nvfp4_status st = device_info(&dev);
  if (st != NVFP4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  double* ssq = reinterpret_cast<double*>(ws + L.scalars);
  float* scales = reinterpret_cast<float*>(ws + L.scalars + 16);
  uint16_t* x = static_cast<uint16_t*>(X);
  uint16_t* r = reinterpret_cast<uint16_t*>(ws + L.r);
  nvfp4_tensor xr{ws + L.xr_codes, ws + L.xr_scales, scales + 0, m, n, NVFP4_SCALE_MMA, 0};
  nvfp4_tensor xc{ws + L.xc_codes, ws + L.xc_scales, scales + 1, n, m, NVFP4_SCALE_MMA, 0};
  nvfp4_tensor rr{ws + L.rr_codes, ws + L.rr_scales, scales + 2, m, m, NVFP4_SCALE_MMA, 0};
  const int grid_x = (int)std::min<int64_t>(m, (int64_t)dev->sm_count * 8);
  cudaError_t e;
  if (normalize) {
    e = cudaMemsetAsync(ssq, 0, sizeof(double), s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(sum of squares)");
    nvfp4::ns::sumsq_kernel<<<grid_x, nvfp4::ns::kThreads, 0, s>>>(static_cast<const uint16_t*>(G), m, n, ldg, ssq);
    nvfp4::ns::normalize_kernel<<<grid_x, nvfp4::ns::kThreads, 0, s>>>(static_cast<const uint16_t*>(G), ldg, x, ldx, m,
                                                                        n, ssq, norm_out);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "normalisation launch");
  } else if (G != X) {
    e = cudaMemcpy2DAsync(X, (size_t)ldx * 2, G, (size_t)ldg * 2, (size_t)n * 2, (size_t)m, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy2DAsync(G -> X)");
  }
  const nvfp4_quant_opts rne{};
  void* qws = ws + L.quant_ws;
  const int grid_r = (int)std::min<int64_t>(m, (int64_t)dev->sm_count * 8);
  for (int32_t it = 0; it < iters; ++it) {
    if ((st = nvfp4_quantize(X, m, n, ldx, &rne, &xr, &xc, qws, kWorkspaceBytes, stream)) != NVFP4_OK) return st;
    nvfp4::ns::identity_kernel<<<grid_r, nvfp4::ns::kThreads, 0, s>>>(r, m, m);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "identity launch");
    if ((st = gemm_impl(&xr, &xr, r, m, NVFP4_OUT_BF16, -1.0f, 1, nullptr, 0u, stream)) != NVFP4_OK) return st;
    if ((st = nvfp4_quantize(r, m, m, m, &rne, &rr, nullptr, qws, kWorkspaceBytes, stream)) != NVFP4_OK) return st;
    if ((st = gemm_impl(&rr, &xc, X, ldx, NVFP4_OUT_BF16, 0.5f, 1, nullptr, 0u, stream)) != NVFP4_OK) return st;
  }
  return NVFP4_OK;
}

}  // extern "C"

namespace {

bool rank_ok(int32_t rank) { return rank >= 16 && rank <= nvfp4::lowrank::kMaxRank && rank % 16 == 0; }

// Tensor map of a row-major BF16 matrix [outer x inner] (row stride ld elements) for
// the projection: boxes of box_outer rows x 64 elements (128 bytes), 128-byte swizzle;
// a box reaching past `inner` is zero-filled.
nvfp4_status make_bf16_box_map(CUtensorMap* map, const void* X, int64_t inner, int64_t outer, int64_t ld,
                               uint32_t box_outer) {
  PFN_cuTensorMapEncodeTiled_v12000 encode;
  nvfp4_status st = get_encoder(&encode);
  if (st != NVFP4_OK) return st;
  const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 2u};
  const cuuint32_t box[2] = {64u, box_outer};
  const cuuint32_t estr[2] = {1u, 1u};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(X), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled(projection operand) failed (%d)", (int)r);
  return NVFP4_OK;
}

template <int RT, bool BT>
cudaError_t launch_project(const CUtensorMap& am, const CUtensorMap& bm, int64_t units, int32_t chunks, int grid,
                           uint16_t* u, int64_t ldu, const float* sa, const float* sb, cudaStream_t s) {
  static bool done[kMaxDevices] = {};
  static std::mutex m;
  auto kernel = nvfp4::lowrank::lowrank_project_kernel<RT, BT>;
  cudaError_t e = ensure_smem(kernel, nvfp4::lowrank::kProjSmemBytes, done, m);
  if (e != cudaSuccess) return e;
  kernel<<<grid, nvfp4::lowrank::kProjThreads, nvfp4::lowrank::kProjSmemBytes, s>>>(am, bm, units, chunks, u, ldu, sa,
                                                                                    sb);
  return cudaGetLastError();
}

template <int RT>
cudaError_t dispatch_project(bool bt, const CUtensorMap& am, const CUtensorMap& bm, int64_t units, int32_t chunks,
                             int grid, uint16_t* u, int64_t ldu, const float* sa, const float* sb, cudaStream_t s) {
  return bt ? launch_project<RT, true>(am, bm, units, chunks, grid, u, ldu, sa, sb, s)
            : launch_project<RT, false>(am, bm, units, chunks, grid, u, ldu, sa, sb, s);
}

template <int KS, bool CT>
cudaError_t launch_expand(uint16_t* y, int64_t ldy, const uint16_t* u, int64_t ldu, const uint16_t* c, int64_t ldc,
                          int64_t M, int64_t N, int sm_count, cudaStream_t s) {
  static bool done[kMaxDevices] = {};
  static std::mutex m;
  auto kernel = nvfp4::lowrank::lowrank_expand_kernel<KS, CT>;
  constexpr int smem = nvfp4::lowrank::exp_smem_bytes<KS>();
  cudaError_t e = ensure_smem(kernel, smem, done, m);
  if (e != cudaSuccess) return e;
  const int64_t tiles_n = N / nvfp4::lowrank::kExpTile;
  const int64_t tiles = (M / nvfp4::lowrank::kExpTile) * tiles_n;
  const int grid = (int)std::min<int64_t>(tiles, sm_count);
  kernel<<<grid, nvfp4::lowrank::kExpThreads, smem, s>>>(y, ldy, u, ldu, c, ldc, (int32_t)tiles_n, (int32_t)tiles);
  return cudaGetLastError();
}

template <int KS>
cudaError_t dispatch_expand(bool ct, uint16_t* y, int64_t ldy, const uint16_t* u, int64_t ldu, const uint16_t* c,
                            int64_t ldc, int64_t M, int64_t N, int sm_count, cudaStream_t s) {
  return ct ? launch_expand<KS, true>(y, ldy, u, ldu, c, ldc, M, N, sm_count, s)
            : launch_expand<KS, false>(y, ldy, u, ldu, c, ldc, M, N, sm_count, s);
}

}  // namespace

extern "C" {

nvfp4_status nvfp4_lora_residual(const void* W, int64_t N, int64_t K, int64_t ldw, const void* L, int64_t ldl,
                                 const void* R, int64_t ldr, int32_t rank, void* W_res, int64_t ldo, void* stream) {
  if (!rank_ok(rank)) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "rank %d is not 16, 32, 48 or 64", rank);
  if (N < 0 || K < 0) return fail(NVFP4_ERR_INVALID_ARG, "negative extent");
  if (K % 8) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "K %lld is not a multiple of 8", (long long)K);
  if (N == 0 || K == 0) return NVFP4_OK;
  if (!W || !L || !R || !W_res) return fail(NVFP4_ERR_INVALID_ARG, "NULL buffer");
  if (ldw < K || ldr < K || ldo < K || ldl < rank) return fail(NVFP4_ERR_INVALID_ARG, "leading dimension too small");
  if (!aligned16(W) || !aligned16(R) || !aligned16(W_res) || ldw % 8 || ldr % 8 || ldo % 8 ||
      reinterpret_cast<uintptr_t>(L) % 2)
    return fail(NVFP4_ERR_MISALIGNED, "W, R and W_res rows must be 16-byte aligned");
  const int64_t per_row = ceil_div(K / 8, nvfp4::lowrank::kResidualThreads);
  const dim3 grid((unsigned)per_row, (unsigned)std::min<int64_t>(ceil_div(N, nvfp4::lowrank::kResRows), 65535));
  nvfp4::lowrank::lora_residual_kernel<<<grid, nvfp4::lowrank::kResidualThreads, 0,
                                         static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(W), ldw, static_cast<const uint16_t*>(L), ldl, static_cast<const uint16_t*>(R),
      ldr, static_cast<uint16_t*>(W_res), ldo, N, K, rank);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "lora residual launch");
}

}  // extern "C"

namespace {
nvfp4_status lowrank_project_impl(const void* A, int64_t M, int64_t K, int64_t lda, const void* B, int64_t ldb,
                                  int32_t b_trans, int32_t rank, const float* sa, const float* sb, void* U,
                                  int64_t ldu, void* stream) {
  if (!rank_ok(rank)) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "rank %d is not 16, 32, 48 or 64", rank);
  if (M < 0 || K < 0) return fail(NVFP4_ERR_INVALID_ARG, "negative extent");
  if (M % nvfp4::lowrank::kProjUnit || K % nvfp4::lowrank::kProjKc || K == 0)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "projection needs M %% 16 == 0 and K a positive multiple of 64");
  if (K / nvfp4::lowrank::kProjKc > INT32_MAX) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "K above 2^37");
  if (M == 0) return NVFP4_OK;
  if (!A || !B || !U) return fail(NVFP4_ERR_INVALID_ARG, "NULL buffer");
  if ((sa == nullptr) != (sb == nullptr)) return fail(NVFP4_ERR_INVALID_ARG, "give both tensor scales or neither");
  if (lda < K || ldu < rank || ldb < (b_trans ? (int64_t)rank : K))
    return fail(NVFP4_ERR_INVALID_ARG, "leading dimension too small");
  if (!aligned16(A) || !aligned16(B) || !aligned16(U) || lda % 8 || ldb % 8 || ldu % 8)
    return fail(NVFP4_ERR_MISALIGNED, "A, B and U rows must be 16-byte aligned");
  DeviceInfo* dev;
  nvfp4_status st = device_info(&dev);
  if (st != NVFP4_OK) return st;
  const bool bt = b_trans != 0;
  CUtensorMap am, bm;
  if ((st = make_bf16_box_map(&am, A, K, M, lda, nvfp4::lowrank::kProjUnit)) != NVFP4_OK) return st;
  // B as [r x K]: boxes of r rows x 64 K; B as [K x r]: boxes of 64 K-rows x 64 columns
  if ((st = bt ? make_bf16_box_map(&bm, B, rank, K, ldb, (uint32_t)nvfp4::lowrank::kProjKc)
               : make_bf16_box_map(&bm, B, K, rank, ldb, (uint32_t)rank)) != NVFP4_OK)
    return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint16_t* u = static_cast<uint16_t*>(U);
  const int64_t units = M / nvfp4::lowrank::kProjUnit;
  const int64_t chunk_cols = (int64_t)nvfp4::lowrank::kProjKc *
                             (bt ? nvfp4::lowrank::proj_halves<true>() : nvfp4::lowrank::proj_halves<false>());
  const int32_t chunks = (int32_t)((K + chunk_cols - 1) / chunk_cols);   // a last half-chunk reads zeros past K
  const int grid = (int)std::min<int64_t>(units, dev->sm_count);
  cudaError_t e;
  switch (rank / 8) {
    case 2: e = dispatch_project<2>(bt, am, bm, units, chunks, grid, u, ldu, sa, sb, s); break;
    case 4: e = dispatch_project<4>(bt, am, bm, units, chunks, grid, u, ldu, sa, sb, s); break;
    case 6: e = dispatch_project<6>(bt, am, bm, units, chunks, grid, u, ldu, sa, sb, s); break;
    default: e = dispatch_project<8>(bt, am, bm, units, chunks, grid, u, ldu, sa, sb, s); break;
  }
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "low-rank projection launch");
}
}  // namespace

extern "C" {

nvfp4_status nvfp4_lowrank_project(const void* A, int64_t M, int64_t K, int64_t lda, const void* B, int64_t ldb,
                                   int32_t b_trans, int32_t rank, void* U, int64_t ldu, void* stream) {
  return lowrank_project_impl(A, M, K, lda, B, ldb, b_trans, rank, nullptr, nullptr, U, ldu, stream);
}

nvfp4_status nvfp4_lowrank_project_scaled(const void* A, int64_t M, int64_t K, int64_t lda, const void* B,
                                          int64_t ldb, int32_t b_trans, int32_t rank, const float* scale_a,
                                          const float* scale_b, void* U, int64_t ldu, void* stream) {
  if (!scale_a || !scale_b) return fail(NVFP4_ERR_INVALID_ARG, "scale_a or scale_b is NULL");
  return lowrank_project_impl(A, M, K, lda, B, ldb, b_trans, rank, scale_a, scale_b, U, ldu, stream);
}

nvfp4_status nvfp4_lowrank_expand_add(void* Y, int64_t M, int64_t N, int64_t ldy, const void* U, int64_t ldu,
                                      const void* C, int64_t ldc, int32_t c_trans, int32_t rank, void* stream) {
  if (!rank_ok(rank)) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "rank %d is not 16, 32, 48 or 64", rank);
  if (M < 0 || N < 0) return fail(NVFP4_ERR_INVALID_ARG, "negative extent");
  if (M % nvfp4::lowrank::kExpTile || N % nvfp4::lowrank::kExpTile)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "expansion needs M %% 128 == 0 and N %% 128 == 0");
  if (M == 0 || N == 0) return NVFP4_OK;
  if (!Y || !U || !C) return fail(NVFP4_ERR_INVALID_ARG, "NULL buffer");
  if (ldy < N || ldu < rank || ldc < (c_trans ? N : (int64_t)rank))
    return fail(NVFP4_ERR_INVALID_ARG, "leading dimension too small");
  if (!aligned16(Y) || !aligned16(U) || !aligned16(C) || ldy % 8 || ldu % 8 || ldc % 8)
    return fail(NVFP4_ERR_MISALIGNED, "Y, U and C rows must be 16-byte aligned");
  if ((M / nvfp4::lowrank::kExpTile) * (N / nvfp4::lowrank::kExpTile) > INT32_MAX)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "expansion has more than 2^31 tiles");
  DeviceInfo* dev;
  nvfp4_status st = device_info(&dev);
  if (st != NVFP4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint16_t* y = static_cast<uint16_t*>(Y);
  const uint16_t* u = static_cast<const uint16_t*>(U);
  const uint16_t* c = static_cast<const uint16_t*>(C);
  const bool ct = c_trans != 0;
  const int sms = dev->sm_count;
  cudaError_t e;
  switch (rank / 16) {
    case 1: e = dispatch_expand<1>(ct, y, ldy, u, ldu, c, ldc, M, N, sms, s); break;
    case 2: e = dispatch_expand<2>(ct, y, ldy, u, ldu, c, ldc, M, N, sms, s); break;
    case 3: e = dispatch_expand<3>(ct, y, ldy, u, ldu, c, ldc, M, N, sms, s); break;
    default: e = dispatch_expand<4>(ct, y, ldy, u, ldu, c, ldc, M, N, sms, s); break;
  }
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "low-rank expansion launch");
}

}  // extern "C"

namespace {

// Arguments of the low-rank branch of a LoRA-SVD call, checked before the NVFP4 part
// launches anything: rows x cols is the output (Y or dX), inner the projection's
// contraction length (K or N).
nvfp4_status lora_precheck(const nvfp4_tensor* Wq, const void* L, const void* R, int32_t rank, const void* U,
                           int64_t rows, int64_t cols, int64_t inner, int64_t ld_in, int64_t ld_out) {
  if (!rank_ok(rank)) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "rank %d is not 16, 32, 48 or 64", rank);
  if (!Wq) return fail(NVFP4_ERR_INVALID_ARG, "the quantised residual weight is NULL");
  if (!L || !R || !U) return fail(NVFP4_ERR_INVALID_ARG, "L, R or U is NULL");
  if (!aligned16(L) || !aligned16(R) || !aligned16(U)) return fail(NVFP4_ERR_MISALIGNED, "L, R and U must be 16-byte aligned");
  if (rows % nvfp4::lowrank::kExpTile || cols % nvfp4::lowrank::kExpTile || inner % nvfp4::lowrank::kProjKc ||
      inner == 0)
    return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "LoRA-SVD needs the output extents %% 128 and the inner extent %% 64");
  if (ld_in % 8 || ld_out % 8) return fail(NVFP4_ERR_MISALIGNED, "input and output rows must be 16-byte aligned");
  return NVFP4_OK;
}

}  // namespace

extern "C" {

nvfp4_status nvfp4_lora_linear_fwd(const void* X, int64_t M, int64_t K, int64_t ldx, const nvfp4_tensor* Wq_res_row,
                                   const void* L, const void* R, int32_t rank, void* Y, int64_t ldy,
                                   nvfp4_tensor* Xq_row, nvfp4_tensor* Xq_col, uint32_t rht_signs, void* U,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  nvfp4_status st = lora_precheck(Wq_res_row, L, R, rank, U, M, Wq_res_row ? Wq_res_row->rows : 0, K, ldx, ldy);
  if (st != NVFP4_OK) return st;
  if ((st = check_tensor(Wq_res_row, "Wq_res_row")) != NVFP4_OK) return st;
  if (!Xq_row) return fail(NVFP4_ERR_INVALID_ARG, "Xq_row is NULL");
  if (Wq_res_row->cols != K) return fail(NVFP4_ERR_INVALID_ARG, "Wq_res_row.cols != K");
  if (M < 256) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "the fused LoRA-SVD linear needs M >= 256");
  nvfp4_quant_opts o{};
  o.rht_col = Xq_col != nullptr;
  o.rht_signs = rht_signs;
  if ((st = nvfp4_quantize(X, M, K, ldx, &o, Xq_row, Xq_col, workspace, workspace_bytes, stream)) != NVFP4_OK)
    return st;
  // U' = BF16(X R^T / (S_X S_W)), then Y = BF16(S_X S_W (Q(X) Q(W_res)^T + U' L^T)) in one GEMM
  if ((st = lowrank_project_impl(X, M, K, ldx, R, K, 0, rank, Xq_row->tensor_scale, Wq_res_row->tensor_scale, U,
                                 rank, stream)) != NVFP4_OK)
    return st;
  return nvfp4_gemm_lowrank(Xq_row, Wq_res_row, U, rank, L, rank, rank, Y, ldy, stream);
}

nvfp4_status nvfp4_lora_linear_dgrad(const void* dY, int64_t M, int64_t N, int64_t ldy, const nvfp4_tensor* Wq_res_col,
                                     const void* L, const void* Rt, int32_t rank, void* dX, int64_t ldx,
                                     nvfp4_tensor* dYq_row, nvfp4_tensor* dYq_col, uint64_t seed, uint64_t offset,
                                     uint32_t rht_signs, void* U, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  nvfp4_status st = lora_precheck(Wq_res_col, L, Rt, rank, U, M, Wq_res_col ? Wq_res_col->rows : 0, N, ldy, ldx);
  if (st != NVFP4_OK) return st;
  if ((st = check_tensor(Wq_res_col, "Wq_res_col")) != NVFP4_OK) return st;
  if (!dYq_row) return fail(NVFP4_ERR_INVALID_ARG, "dYq_row is NULL");
  if (Wq_res_col->cols != N) return fail(NVFP4_ERR_INVALID_ARG, "Wq_res_col.cols != N");
  if (M < 256) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "the fused LoRA-SVD linear needs M >= 256");
  nvfp4_quant_opts o{};
  o.stochastic = 1;
  o.rht_col = dYq_col != nullptr;
  o.seed = seed;
  o.offset = offset;
  o.rht_signs = rht_signs;
  if ((st = nvfp4_quantize(dY, M, N, ldy, &o, dYq_row, dYq_col, workspace, workspace_bytes, stream)) != NVFP4_OK)
    return st;
  // U' = BF16(dY L / (S_dY S_W)), then dX = BF16(S_dY S_W (Q(dY) Q(W_res) + U' R)) in one GEMM
  if ((st = lowrank_project_impl(dY, M, N, ldy, L, rank, 1, rank, dYq_row->tensor_scale, Wq_res_col->tensor_scale,
                                 U, rank, stream)) != NVFP4_OK)
    return st;
  return nvfp4_gemm_lowrank(dYq_row, Wq_res_col, U, rank, Rt, rank, rank, dX, ldx, stream);
}

nvfp4_status nvfp4_quantize_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                    const nvfp4_quant_opts* opts, nvfp4_tensor* out_row, nvfp4_tensor* out_col,
                                    void* stream) {
  // The scratch this call needs must fit the fixed array; it does not grow with
  // the tensor (three amax accumulators), but the check keeps the limit explicit.
  const size_t need = kWorkspaceBytes;
  if (need > kNoAllocScratchBytes)
    return fail(NVFP4_ERR_WORKSPACE, "quantize needs %zu bytes of scratch, the fixed scratch holds %zu", need,
                kNoAllocScratchBytes);
  void* scratch = nullptr;
  nvfp4_status st = noalloc_scratch(&scratch);
  if (st != NVFP4_OK) return st;
  // the quantiser clears the accumulators it uses at the start of every call
  return nvfp4_quantize(x, rows, cols, ld, opts, out_row, out_col, scratch, kNoAllocScratchBytes, stream);
}

nvfp4_status nvfp4_check_conversions(unsigned long long* counts, uint64_t n_sr, void* stream) {
  if (!counts) return fail(NVFP4_ERR_INVALID_ARG, "counts is NULL");
  if (!aligned16(counts)) return fail(NVFP4_ERR_MISALIGNED, "counts is not 16-byte aligned");
  DeviceInfo* dev;
  nvfp4_status st = device_info(&dev);
  if (st != NVFP4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(counts, 0, 3 * sizeof(unsigned long long), s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(counts)");
  nvfp4::check_conversions_kernel<<<dev->sm_count * 8, 256, 0, s>>>(counts, n_sr);
  e = cudaGetLastError();
  return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "check_conversions launch");
}

nvfp4_status nvfp4_get_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned word = 0;
  e = cudaMemcpyFromSymbol(&word, nvfp4::g_error_word, sizeof(word));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (word) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(nvfp4::g_error_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
    if (word & nvfp4::kErrTimeout) return fail(NVFP4_ERR_TIMEOUT, "a device-side wait exceeded its time limit");
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pending CUDA error");
  return NVFP4_OK;
}

}  // extern "C"
