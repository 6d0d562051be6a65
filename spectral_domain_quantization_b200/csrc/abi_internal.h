// Internal building blocks shared by the C ABI entry points.
#pragma once

#include "abi_common.h"

namespace metis {

metis_status validate_dense(const void* X, int dtype, int64_t rows, int64_t cols, int64_t ld);

// Workspace the quantizer needs for `out`.
size_t quantize_workspace(const metis_fp4_tensor* out);

// Enqueue the FP4 quantization of X (axis 1: blocks along columns; 0: along
// rows) into `out`.  amax_bits_in: optional precomputed NVFP4 tensor max
// (float bits) on the device; r_tap: optional float32 copy of the quantizer's
// input (rows x cols, row-major).
metis_status enqueue_quantize(const void* X, int dtype, int64_t rows, int64_t cols, int64_t ld,
                              int axis, const float* sub_col, const metis_fp4_tensor* out,
                              const unsigned* amax_bits_in, float* r_tap, Carver& ws,
                              cudaStream_t s);

}  // namespace metis
