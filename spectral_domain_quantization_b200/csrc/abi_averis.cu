// C ABI: averis_split (see include/metis.h).
//
// Source: retelling of arXiv 2603.10444, Averis paragraphs (mean over all
// rows, broadcast subtraction, separate FP4 quantization of the mean vector
// and of the mean-free residual; the same split of the output gradient in the
// backward pass).
#include "abi_common.h"
#include "abi_internal.h"
#include "averis.h"
#include "common.cuh"
#include "kernels.h"

using namespace metis;

namespace {

struct AverisBuffers {
  double* psum;
  float* pmin;
  float* pmax;
  unsigned* amax;
};

AverisBuffers carve_averis(int64_t nchunks, int64_t n, Carver& ws) {
  AverisBuffers b;
  b.psum = ws.take<double>(static_cast<size_t>(nchunks) * n);
  b.pmin = ws.take<float>(static_cast<size_t>(nchunks) * n);
  b.pmax = ws.take<float>(static_cast<size_t>(nchunks) * n);
  b.amax = ws.take<unsigned>(1);
  return b;
}

}  // namespace

extern "C" metis_status averis_split(const void* X, int32_t dtype, int64_t m, int64_t n, int64_t ld, int32_t fmt,
                                     float* mean, metis_fp4_tensor* mean_q, metis_fp4_tensor* R_rows,
                                     metis_fp4_tensor* R_cols, float* R_f32, void* workspace,
                                     size_t* workspace_bytes, int32_t* dev_status, void* stream) {
  if (!workspace_bytes || !mean) return METIS_ERR_NULL;
  METIS_TRY(validate_dense(X, dtype, m, n, ld));
  if (!valid_fmt(fmt)) return METIS_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(mean) & 15u) != 0) return METIS_ERR_ALIGN;
  if (mean_q) METIS_TRY(check_fp4(mean_q, 1, n, fmt));
  if (R_rows) METIS_TRY(check_fp4(R_rows, m, n, fmt));
  if (R_cols) METIS_TRY(check_fp4(R_cols, n, m, fmt));
  const int sms = device_sm_count();
  const int64_t nchunks = colstats_chunks(X, dtype, m, n, ld, sms);
  size_t need;
  {
    Carver c(nullptr);
    carve_averis(nchunks, n, c);
    need = c.used;
    if (mean_q) need += quantize_workspace(mean_q);
    if (R_rows) need += quantize_workspace(R_rows);
    if (R_cols) need += quantize_workspace(R_cols);
  }
  if (!workspace) {
    *workspace_bytes = need;
    return METIS_OK;
  }
  if (*workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return METIS_ERR_WORKSPACE;
  if (!device_is_sm100()) return METIS_ERR_UNSUPPORTED;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  Carver ws(workspace);
  const AverisBuffers b = carve_averis(nchunks, n, ws);
  launch_colstats(X, dtype, m, n, ld, sms, b.psum, b.pmin, b.pmax, mean, b.amax, dev_status, s);
  if (mean_q) METIS_TRY(enqueue_quantize(mean, METIS_F32, 1, n, n, 1, nullptr, mean_q, nullptr, nullptr, ws, s));
  bool tapped = false;
  if (R_rows) {
    METIS_TRY(enqueue_quantize(X, dtype, m, n, ld, 1, mean, R_rows, fmt == METIS_NVFP4 ? b.amax : nullptr, R_f32, ws,
                               s));
    tapped = R_f32 != nullptr;
  }
  if (R_cols) {
    METIS_TRY(enqueue_quantize(X, dtype, m, n, ld, 0, mean, R_cols, fmt == METIS_NVFP4 ? b.amax : nullptr,
                               tapped ? nullptr : R_f32, ws, s));
    tapped = R_f32 != nullptr;
  }
  if (R_f32 && !tapped) launch_residual_tap(X, dtype, m, n, ld, mean, R_f32, device_sm_count(), s);
  return launch_status();
}
