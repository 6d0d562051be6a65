// Host-side helpers of the C ABI and the entry points that need no kernels.
#include <atomic>
#include <cstddef>
#include <cstdio>
#include <mutex>

#include "abi_common.h"
#include "common.cuh"

// The Python binding mirrors these structs field by field (ctypes); a layout
// change must change both sides.
static_assert(sizeof(metis_fp4_tensor) == 64 && offsetof(metis_fp4_tensor, outer) == 8 &&
                  offsetof(metis_fp4_tensor, codes) == 24 && offsetof(metis_fp4_tensor, inner_sum) == 56,
              "metis_fp4_tensor layout");
static_assert(sizeof(metis_operand) == 48 && offsetof(metis_operand, k) == 8 && offsetof(metis_operand, P) == 16 &&
                  offsetof(metis_operand, S) == 32 && offsetof(metis_operand, flags) == 40,
              "metis_operand layout");

namespace metis {

namespace {
constexpr int kMaxDevices = 64;
// Per-device properties, filled on first use.  g_major is written before
// g_sm_count is published (release), and readers check g_sm_count first
// (acquire), so a thread that sees the count also sees the major version.
std::atomic<int> g_sm_count[kMaxDevices];
std::atomic<int> g_major[kMaxDevices];
std::once_flag g_driver_once;
// signature of cuTensorMapEncodeTiled (driver API, CUDA 12.0+)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

void fill_props(int dev) {
  if (dev < 0 || dev >= kMaxDevices || g_sm_count[dev].load(std::memory_order_acquire) != 0) return;
  int sms = 0, major = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  g_major[dev].store(major, std::memory_order_relaxed);
  g_sm_count[dev].store(sms, std::memory_order_release);
}
}  // namespace

int device_sm_count() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  fill_props(dev);
  const int sms = g_sm_count[dev].load(std::memory_order_acquire);
  return sms > 0 ? sms : 148;
}

bool device_is_sm100() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return false;
  fill_props(dev);
  if (g_sm_count[dev].load(std::memory_order_acquire) == 0) return false;
  return g_major[dev].load(std::memory_order_relaxed) == 10;
}

CUresult encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank,
                           const void* gaddr, const uint64_t* dims, const uint64_t* strides_bytes,
                           const uint32_t* box, CUtensorMapSwizzle swizzle) {
  std::call_once(g_driver_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  if (!g_encode) return CUDA_ERROR_NOT_SUPPORTED;
  uint32_t elem_strides[5] = {1, 1, 1, 1, 1};
  return g_encode(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void*>(gaddr),
                  reinterpret_cast<const cuuint64_t*>(dims),
                  reinterpret_cast<const cuuint64_t*>(strides_bytes), box, elem_strides,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

metis_status check_fp4(const metis_fp4_tensor* t, int64_t outer, int64_t inner, int fmt) {
  if (!t || !t->codes || !t->scales) return METIS_ERR_NULL;
  if (!valid_fmt(t->fmt) || t->fmt != fmt) return METIS_ERR_ARG;
  if (t->outer != outer || t->inner != inner) return METIS_ERR_SHAPE;
  if (outer <= 0 || inner <= 0 || inner % 32 != 0) return METIS_ERR_SHAPE;
  if (t->fmt == METIS_NVFP4 && !t->tensor_scale) return METIS_ERR_NULL;
  if (!aligned16(t->codes) || !aligned16(t->scales)) return METIS_ERR_ALIGN;
  return METIS_OK;
}

namespace {
thread_local char g_last_error[256] = "";
}

metis_status fail(metis_status st, const char* where, const char* detail) {
  snprintf(g_last_error, sizeof(g_last_error), "%s%s%s", where ? where : "", detail ? ": " : "",
           detail ? detail : "");
  return st;
}

// The dynamic shared-memory limit is a per-device attribute of a kernel:
// the cache of limits already set is keyed by (kernel, device).
bool ensure_smem(const void* kernel, size_t bytes) {
  static std::mutex mu;
  static const void* keys[128];
  static int devs[128];
  static size_t vals[128];
  static int count = 0;
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(mu);
  int slot = -1;
  for (int i = 0; i < count; ++i)
    if (keys[i] == kernel && devs[i] == dev) slot = i;
  if (slot >= 0 && vals[slot] >= bytes) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) !=
      cudaSuccess)
    return false;
  if (slot < 0 && count < 128) {
    slot = count++;
    keys[slot] = kernel;
    devs[slot] = dev;
  }
  if (slot >= 0) vals[slot] = bytes;
  return true;
}

metis_status step_status(const char* where) {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return METIS_OK;
  return fail(METIS_ERR_CUDA, where, cudaGetErrorString(e));
}

metis_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return METIS_OK;
  return fail(METIS_ERR_CUDA, "kernel launch", cudaGetErrorString(e));
}

}  // namespace metis

extern "C" {

size_t metis_fp4_codes_bytes(int64_t outer, int64_t inner) {
  if (outer <= 0 || inner <= 0) return 0;
  return static_cast<size_t>(outer) * static_cast<size_t>((inner + 1) / 2);
}

size_t metis_fp4_scales_bytes(int32_t fmt, int64_t outer, int64_t inner) {
  if (outer <= 0 || inner <= 0 || !metis::valid_fmt(fmt)) return 0;
  return static_cast<size_t>(metis::tc_scale_rows(outer)) *
         static_cast<size_t>(metis::tc_scale_cols(fmt, inner));
}

const char* metis_status_string(int32_t status) {
  switch (status) {
    case METIS_OK: return "ok";
    case METIS_ERR_NULL: return "a required pointer is NULL";
    case METIS_ERR_SHAPE: return "invalid shape";
    case METIS_ERR_ALIGN: return "misaligned pointer or leading dimension";
    case METIS_ERR_UNSUPPORTED: return "unsupported device or option";
    case METIS_ERR_WORKSPACE: return "workspace too small or misaligned";
    case METIS_ERR_CUDA: return "CUDA error";
    case METIS_ERR_ARG: return "invalid argument";
    default: return "unknown status";
  }
}

int32_t metis_device_supported(void) { return metis::device_is_sm100() ? 1 : 0; }

const char* metis_last_error(void) { return metis::g_last_error; }

}  // extern "C"

namespace {

// One thread waits, with the kernels' own bounded wait, on a barrier phase
// that nothing completes; the timeout must end the wait and be reported.
__global__ void wait_selftest_kernel(uint64_t limit_ns, int32_t* dev_status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  abort_flag = 0;
  metis::mbar_init(&bar, 1);
  metis::fence_barrier_init();
  if (!metis::mbar_wait_for(&bar, 0, &abort_flag, limit_ns)) metis::report(dev_status, METIS_DEV_TIMEOUT);
}

}  // namespace

extern "C" metis_status metis_selftest_wait_timeout(uint64_t limit_ns, int32_t* dev_status, void* stream) {
  if (!dev_status) return METIS_ERR_NULL;
  if (limit_ns == 0 || limit_ns > 1000000000ull) return METIS_ERR_ARG;
  if (!metis::device_is_sm100()) return METIS_ERR_UNSUPPORTED;
  wait_selftest_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, dev_status);
  return metis::launch_status();
}
