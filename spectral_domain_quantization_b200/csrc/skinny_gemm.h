// Interface of the tall-skinny tcgen05 bf16 GEMM (skinny_gemm.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/metis.h"

namespace metis {

struct SkinnyParams {
  int mode;
  int64_t rows_out, K;
  int lp, xparts, aparts, nmma;
  int cs;                   // CTAs per cluster = K slices per 128-row tile
  int64_t ksteps_per_split, total_ksteps;
  float* out;
  __nv_bfloat16* outT;
  int64_t ldo;
  int32_t* dev_status;
};

struct SkinnyCall {
  int mode;               // 0: Y = A X (m x lp); 1: Y = A^T X (n x lp)
  int64_t m, n, lda;      // A is m x n bf16 (row-major, leading dimension lda)
  const void* A[2];       // bf16 parts of A (one, or hi and lo of an fp32 A)
  int aparts;
  const void* Xt;         // bf16 [xparts * lp][ldx], K = n (mode 0) or m (mode 1) used
  int64_t ldx;            // multiple of 8 (16-byte rows)
  int xparts;
  int lp;                 // multiple of 16, xparts * lp <= 256
  int cs;                 // 1, 2, 4 or 8 (skinny_cluster)
  float* out;             // optional Y, [rows_out][lp] float32
  __nv_bfloat16* outT;    // optional Y^T as bf16 hi / lo: [2 lp][ldo], hi rows 0..lp-1
  int64_t ldo;
  int32_t* dev_status;
};

// 128-row output tiles of a product with rows_out rows.
int skinny_tiles(int64_t rows_out);
// CTAs per cluster (K slices per tile) for a product of rows_out rows and
// contraction length K on `sms` SMs.
int skinny_cluster(int64_t rows_out, int64_t K, int sms);
metis_status run_skinny_gemm(const SkinnyCall& c, cudaStream_t s);

}  // namespace metis
