// Host-side helpers of the C ABI: argument checks, workspace carving, device
// properties, driver entry points.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/metis.h"

namespace metis {

// Bump allocator over the caller's workspace.  In query mode (base == NULL)
// it only adds up the sizes.  Every slot is 256-byte aligned.
struct Carver {
  char* base;
  size_t used = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <class T>
  T* take(size_t count) {
    const size_t bytes = (count * sizeof(T) + 255) & ~static_cast<size_t>(255);
    T* p = base ? reinterpret_cast<T*>(base + used) : nullptr;
    used += bytes;
    return p;
  }
};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t dtype_size(int dt) { return dt == METIS_BF16 ? 2 : 4; }
inline bool valid_dtype(int dt) { return dt == METIS_BF16 || dt == METIS_F32; }
inline bool valid_fmt(int f) { return f == METIS_MXFP4 || f == METIS_NVFP4; }

// Number of SMs of the current device (cached per device).
int device_sm_count();
// 1 when the current device is compute capability 10.x.
bool device_is_sm100();

// cuTensorMapEncodeTiled through the runtime's driver entry point.
// dims[rank] innermost first; strides_bytes[rank-1] for dims 1..rank-1;
// box[rank] in elements; zero fill out of bounds.
CUresult encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank,
                           const void* gaddr, const uint64_t* dims, const uint64_t* strides_bytes,
                           const uint32_t* box, CUtensorMapSwizzle swizzle);

// Validate a metis_fp4_tensor against an expected shape.
metis_status check_fp4(const metis_fp4_tensor* t, int64_t outer, int64_t inner, int fmt);

// Finish a launch sequence: map a pending CUDA error to METIS_ERR_CUDA.
metis_status launch_status();
// METIS_OK, or METIS_ERR_CUDA naming `where` if a launch or call before it
// failed (a synchronous error such as an invalid launch configuration).
metis_status step_status(const char* where);
// Raise a kernel's dynamic shared-memory limit to at least `bytes` (cached
// per kernel); false if the runtime refuses.
bool ensure_smem(const void* kernel, size_t bytes);
// Record a failure description for metis_last_error(); returns `st`.
metis_status fail(metis_status st, const char* where, const char* detail = nullptr);

}  // namespace metis

#define METIS_TRY(expr)                 \
  do {                                  \
    metis_status _st = (expr);          \
    if (_st != METIS_OK) return _st;    \
  } while (0)
