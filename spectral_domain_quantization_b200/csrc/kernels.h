// Internal launch interface between the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/metis.h"

namespace metis {

// ---- FP4 quantizer -------------------------------------------------------
struct QuantParams {
  const void* X;          // input, row-major
  int dtype;              // METIS_BF16 / METIS_F32
  int64_t ld;             // leading dimension of X (elements)
  const float* sub;       // optional per-column subtraction (length = X's columns)
  int fmt;                // METIS_MXFP4 / METIS_NVFP4
  int64_t outer, inner;   // quantized shape (blocks along inner)
  int64_t ngroups;        // ceil(inner / 64)
  int64_t scale_cols;     // padded scale columns of the tensor-core layout
  uint8_t* codes;
  uint8_t* scales;
  uint8_t* scales_linear;
  float* tensor_scale;    // NVFP4 output s_t
  const unsigned* amax_bits;  // NVFP4 input: tensor max |x| as float bits
  float* partial_sums;    // optional [outer][ngroups] workspace
  float* inner_sum;       // optional output [outer]
  float* r_tap;           // optional float32 copy of the quantized input
  int64_t tap_ld;
};

int64_t quant_groups(int64_t inner);
void launch_amax(const void* X, int dtype, int64_t rows, int64_t cols, int64_t ld, const float* sub,
                 unsigned* out_bits, int num_sms, cudaStream_t s);
// axis 1: blocks along X's columns (outer = rows); axis 0: along rows.
void launch_quantize(const QuantParams& p, int axis, int num_sms, cudaStream_t s);
// The TMA-fed quantizer (quantize_tma.cu) for bf16 X: whether it takes this
// call, and its launch (regroups the partial sums itself).
bool quantize_tma_ok(const QuantParams& p, int axis, int sms);
int64_t quantize_tma_groups(const QuantParams& p, int axis, int sms);
void launch_quantize_tma(QuantParams p, int axis, int sms, int32_t* dev_status, cudaStream_t s);

}  // namespace metis
