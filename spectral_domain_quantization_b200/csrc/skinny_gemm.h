// Interface of the tall-skinny tcgen05 bf16 GEMM (skinny_gemm.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/metis.h"

namespace metis {

struct SkinnyParams {
  int mode;
  int64_t rows_out, K;
  int lp, xparts, aparts, nmma;
  int splits;
  int64_t ksteps_per_split, total_ksteps;
  float* out;
  int32_t* dev_status;
};

struct SkinnyCall {
  int mode;               // 0: out = A X (m x lp); 1: out = A^T X (n x lp)
  int64_t m, n, lda;      // A is m x n bf16 (row-major, leading dimension lda)
  const void* A[2];       // bf16 parts of A (one, or hi and lo of an fp32 A)
  int aparts;
  const void* Xt;         // bf16 [xparts * lp][ldx], K = n (mode 0) or m (mode 1) used
  int64_t ldx;            // multiple of 8 (16-byte rows)
  int xparts;
  int lp;                 // multiple of 16, xparts * lp <= 256
  int splits;
  float* out;             // [splits][rows_out][lp]
  int32_t* dev_status;
};

int skinny_splits(int64_t rows_out, int64_t K, int sms);
metis_status run_skinny_gemm(const SkinnyCall& c, cudaStream_t s);

}  // namespace metis
