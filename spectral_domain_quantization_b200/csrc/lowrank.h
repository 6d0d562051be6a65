// Interface of the low-rank operand builders (lowrank.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/metis.h"

namespace metis {

// Read-only view of one FP4 factor (outer = k, inner = length), or the
// all-ones vector.
struct FactorView {
  int ones;
  int fmt;
  int64_t inner;
  int64_t scale_cols;
  const uint8_t* codes;
  const uint8_t* scales;
  const float* tensor_scale;
};

struct LowRankArgs {
  int64_t M, N;
  int ka, kb;
  int64_t lr_k;             // padded width of LA / LB (multiple of 64)
  FactorView fa;            // F_A (outer ka, inner M)
  FactorView fb;            // F_B (outer kb, inner N)
  const float* s_a;         // S_A (ka) or NULL
  const float* s_b;         // S_B (kb) or NULL
  const float* t1raw;       // R_A P_B, M x kb (row stride t1_ld), or NULL
  int64_t t1_ld;
  const float* t1part;      // or its split-K partial sums (t1_splits x M x kb), summed here
  int t1_splits;
  const float* t1_ts_a;     // tensor scales of that product's operands (NVFP4) or NULL
  const float* t1_ts_b;
  const float* t2raw;       // P_A^T R_B, ka x N (row stride t2_ld)
  int64_t t2_ld;
  const float* cab;         // P_A^T P_B, ka x kb, or NULL
  const float* ts_ra;       // tensor scales of the residuals (NVFP4) or NULL
  const float* ts_rb;
  __nv_bfloat16* la;        // out: M x lr_k
  __nv_bfloat16* lb;        // out: N x lr_k
  // FP4 re-quantized intermediates: T1 (M x kb) in blocks along kb, T2
  // (ka x N) in blocks along ka, each with its own NVFP4 tensor scale
  int requant_t1, requant_t2;
  int fmt;                  // format of the re-quantization (the product's)
  float* t1full;            // M x kb: T1 with every term and S_B (requant_t1)
  unsigned* amax1;          // max |T1| bits (NVFP4), zeroed before the build
  unsigned* amax2;          // max |T2| bits (NVFP4)
};

// Cab = P^_A P^_B^T (ka x kb, tensor scales applied) over the contraction
// of length K: cab_parts(K, sms) partial products (part: that many ka x kb
// floats of scratch), then their sum in a fixed order.  False when the
// kernel's shared memory cannot be granted (nothing is launched).
int cab_parts(int64_t K, int sms);
bool launch_cab(const FactorView& pa, const FactorView& pb, int64_t K, int ka, int kb, float* part, float* cab,
                int sms, cudaStream_t s);
void launch_build_lowrank(const LowRankArgs& a, int sms, cudaStream_t s);
// hi / lo bf16 operands [rows][kp] of deq(U_q) (m rows) and deq(V_q) diag(S)
// (n rows) for the error-compensated residual (fu: U_q, fv: V_q, k factors).
void launch_compensated_operands(const FactorView& fu, const FactorView& fv, int64_t m, int64_t n, int k,
                                 const float* S, int kp, __nv_bfloat16* u_hi, __nv_bfloat16* u_lo,
                                 __nv_bfloat16* w_hi, __nv_bfloat16* w_lo, int sms, cudaStream_t s);


}  // namespace metis
