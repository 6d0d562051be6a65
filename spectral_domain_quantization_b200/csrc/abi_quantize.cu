// C ABI: metis_quantize_fp4 (see include/metis.h for the contract).
#include "abi_common.h"
#include "abi_internal.h"
#include "common.cuh"
#include "kernels.h"

namespace metis {

metis_status validate_dense(const void* X, int dtype, int64_t rows, int64_t cols, int64_t ld) {
  if (!X) return METIS_ERR_NULL;
  if (!valid_dtype(dtype)) return METIS_ERR_ARG;
  if (rows <= 0 || cols <= 0 || ld < cols) return METIS_ERR_SHAPE;
  if (!aligned16(X) || (ld * static_cast<int64_t>(dtype_size(dtype))) % 16 != 0) return METIS_ERR_ALIGN;
  return METIS_OK;
}

size_t quantize_workspace(const metis_fp4_tensor* out) {
  Carver c(nullptr);
  c.take<unsigned>(1);
  if (out->inner_sum) c.take<float>(static_cast<size_t>(out->outer) * quant_groups(out->inner));
  return c.used;
}

metis_status enqueue_quantize(const void* X, int dtype, int64_t rows, int64_t cols, int64_t ld,
                              int axis, const float* sub_col, const metis_fp4_tensor* out,
                              const unsigned* amax_bits_in, float* r_tap, Carver& ws,
                              cudaStream_t s) {
  QuantParams p{};
  p.X = X;
  p.dtype = dtype;
  p.ld = ld;
  p.sub = sub_col;
  p.fmt = out->fmt;
  p.outer = out->outer;
  p.inner = out->inner;
  p.ngroups = quant_groups(p.inner);
  p.scale_cols = tc_scale_cols(p.fmt, p.inner);
  p.codes = out->codes;
  p.scales = out->scales;
  p.scales_linear = out->scales_linear;
  p.tensor_scale = out->tensor_scale;
  p.inner_sum = out->inner_sum;
  p.r_tap = r_tap;
  p.tap_ld = cols;
  unsigned* amax = ws.take<unsigned>(1);
  if (out->inner_sum) p.partial_sums = ws.take<float>(static_cast<size_t>(p.outer) * p.ngroups);
  const int sms = device_sm_count();
  if (cudaMemsetAsync(out->scales, 0, metis_fp4_scales_bytes(p.fmt, p.outer, p.inner), s) != cudaSuccess)
    return METIS_ERR_CUDA;
  if (p.fmt == METIS_NVFP4) {
    if (amax_bits_in) {
      p.amax_bits = amax_bits_in;
    } else {
      if (cudaMemsetAsync(amax, 0, sizeof(unsigned), s) != cudaSuccess) return METIS_ERR_CUDA;
      launch_amax(X, dtype, rows, cols, ld, sub_col, amax, sms, s);
      p.amax_bits = amax;
    }
  }
  launch_quantize(p, axis, sms, s);
  return launch_status();
}

}  // namespace metis

using namespace metis;

extern "C" metis_status metis_quantize_fp4(const void* X, int32_t dtype, int64_t rows,
                                           int64_t cols, int64_t ld, int32_t block_axis,
                                           const float* sub_col, metis_fp4_tensor* out,
                                           void* workspace, size_t* workspace_bytes,
                                           void* stream) {
  if (!out || !workspace_bytes) return METIS_ERR_NULL;
  METIS_TRY(validate_dense(X, dtype, rows, cols, ld));
  if (block_axis != 0 && block_axis != 1) return METIS_ERR_ARG;
  const int64_t outer = block_axis == 1 ? rows : cols;
  const int64_t inner = block_axis == 1 ? cols : rows;
  METIS_TRY(check_fp4(out, outer, inner, out->fmt));
  const size_t need = quantize_workspace(out);
  if (!workspace) {
    *workspace_bytes = need;
    return METIS_OK;
  }
  if (*workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return METIS_ERR_WORKSPACE;
  if (!device_is_sm100()) return METIS_ERR_UNSUPPORTED;
  Carver ws(workspace);
  return enqueue_quantize(X, dtype, rows, cols, ld, block_axis, sub_col, out, nullptr, nullptr, ws,
                          static_cast<cudaStream_t>(stream));
}
