// C ABI: metis_quantize_fp4_noalloc -- the FP4 quantizer for callers that
// cannot hand the library a workspace.
//
// Some callers have no way to obtain scratch memory at the point where they
// quantize: code that must not call cudaMalloc (a runtime that owns every
// device byte through its own arena, a plugin whose host framework forbids
// allocations while it executes, a hot loop that may not block on the
// allocator), or a plain C program that only holds its input and output
// buffers.  For them this entry point keeps its scratch in one fixed array
// compiled into the library, so the only memory the caller provides is the
// input and the FP4 output.
//
// The arithmetic is exactly that of metis_quantize_fp4 (the same kernels are
// enqueued); only where the scratch lives differs.
#include <cuda.h>

#include <mutex>

#include "abi_common.h"
#include "abi_internal.h"
#include "common.cuh"

namespace {

// Every GPU that loads the library holds this array until the process exits.
constexpr size_t kFixedScratchBytes = 2u << 20;  // 2 MiB
__device__ __align__(256) unsigned char g_fixed_scratch[kFixedScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;

// The address is cached per device together with the unique ID of the CUDA
// context it was looked up in: after a context is destroyed and re-created
// (cudaDeviceReset), the library's device code may load at another address,
// so a new context ID means a new lookup.
struct CachedAddr {
  unsigned long long ctx_id;
  void* addr;
};
CachedAddr g_scratch_addr[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
std::once_flag g_ctx_fns_once;
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

// Unique ID of the current context (0 if it cannot be read).
unsigned long long current_ctx_id() {
  std::call_once(g_ctx_fns_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(fn);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (g_ctx_get_current && g_ctx_get_id && g_ctx_get_current(&ctx) == CUDA_SUCCESS && ctx &&
      g_ctx_get_id(ctx, &id) == CUDA_SUCCESS)
    return id;
  return 0;
}

// Device address of the fixed scratch on the current device.  The array's
// name is only a host-side stand-in for it, so the address is looked up with
// that device current and kept for as long as its context lives.
metis_status fixed_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return metis::fail(METIS_ERR_CUDA, "metis_quantize_fp4_noalloc", "no current CUDA device");
  const unsigned long long id = current_ctx_id();
  std::lock_guard<std::mutex> lock(g_mu);
  CachedAddr& c = g_scratch_addr[dev];
  if (!c.addr || id == 0 || c.ctx_id != id) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_fixed_scratch);
    if (e != cudaSuccess || !p)
      return metis::fail(METIS_ERR_CUDA, "metis_quantize_fp4_noalloc: cudaGetSymbolAddress", cudaGetErrorString(e));
    c.addr = p;
    c.ctx_id = current_ctx_id();   // the lookup created the context if there was none
  }
  *out = c.addr;
  return METIS_OK;
}

}  // namespace

using namespace metis;

extern "C" size_t metis_noalloc_scratch_bytes(void) { return kFixedScratchBytes; }

extern "C" metis_status metis_quantize_fp4_noalloc(const void* X, int32_t dtype, int64_t rows, int64_t cols,
                                                   int64_t ld, int32_t block_axis, const float* sub_col,
                                                   metis_fp4_tensor* out, void* stream) {
  if (!out) return METIS_ERR_NULL;
  METIS_TRY(validate_dense(X, dtype, rows, cols, ld));
  if (block_axis != 0 && block_axis != 1) return METIS_ERR_ARG;
  const int64_t outer = block_axis == 1 ? rows : cols;
  const int64_t inner = block_axis == 1 ? cols : rows;
  METIS_TRY(check_fp4(out, outer, inner, out->fmt));
  const size_t need = quantize_workspace(out);
  if (need > kFixedScratchBytes)
    return fail(METIS_ERR_WORKSPACE, "metis_quantize_fp4_noalloc",
                "this size needs more scratch than the library's fixed 2 MiB array (inner sums of "
                "outer x ceil(inner/64) floats); use metis_quantize_fp4 with a workspace");
  if (!device_is_sm100()) return METIS_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  METIS_TRY(fixed_scratch(&scratch));
  // enqueue_quantize zeroes the tensor-maximum word itself and overwrites
  // every inner-sum partial it later reads, so no state leaks between calls
  Carver ws(scratch);
  return enqueue_quantize(X, dtype, rows, cols, ld, block_axis, sub_col, out, nullptr, nullptr, ws,
                          static_cast<cudaStream_t>(stream));
}
