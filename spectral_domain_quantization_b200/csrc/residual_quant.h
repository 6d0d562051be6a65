// Interface of the fused residual + FP4 quantization kernel (residual_quant.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/metis.h"

namespace metis {

struct ResidualParams {
  const void* A;
  int dtype;
  int64_t m, n, lda;
  int kp;                 // k padded to 64 (64 or 128)
  int fmt;
  int mode;               // 0: tensor max of |R| into amax_bits; 1: quantize
  unsigned* amax_bits;
  uint8_t* r_codes;       // blocks along n (outer m, inner n), or NULL
  uint8_t* r_scales;
  int64_t r_scale_cols;
  uint8_t* c_codes;       // blocks along m (outer n, inner m), or NULL
  uint8_t* c_scales;
  int64_t c_scale_cols;
  float* ts_rows;         // NVFP4 tensor scale outputs
  float* ts_cols;
  float* r_tap;           // optional m x n float32 residual
  int32_t* dev_status;
};

struct ResidualOperands {
  const __nv_bfloat16 *u_hi, *u_lo;  // m x kp
  const __nv_bfloat16 *w_hi, *w_lo;  // n x kp, W = V diag(S)
};

// Sign flip of the factors U (m x k) and V (n x k) in place, bf16 hi / lo
// copies of U and V diag(S) padded to kp columns (skipped when u_hi is
// NULL), and the maxima of |U|, |V| into amax[0..1] (skipped when NULL; the
// caller zeroes them first).
void launch_factor_finish(float* U, int64_t m, float* V, int64_t n, int k, const float* sign, const float* S, int kp,
                          __nv_bfloat16* u_hi, __nv_bfloat16* u_lo, __nv_bfloat16* w_hi, __nv_bfloat16* w_lo,
                          unsigned* amax, int sms, cudaStream_t s);
metis_status run_residual_quant(const ResidualParams& p, const ResidualOperands& o, cudaStream_t s);

}  // namespace metis
