// Interface of the block-scaled FP4 GEMM kernel (gemm_fp4.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/metis.h"

namespace metis {

// Kernel parameters (device side).
struct GemmParams {
  int fmt;
  int M, N;
  int num_kt;               // 256-element K tiles
  const uint8_t* sfa;       // A scales, tensor-core layout
  const uint8_t* sfb;
  int64_t sfa_chunks;       // 512-byte scale chunks per 128-row group of A
  int64_t sfb_chunks;
  int64_t sfb_rows;         // padded scale rows of B
  const float* ts_a;        // NVFP4 tensor scales (NULL for MXFP4)
  const float* ts_b;
  int lr_chunks;            // 64-wide bf16 low-rank chunks appended to the K loop
  void* C;
  int c_dtype;
  int64_t ldc;
  int vec_ok;               // 16-byte aligned rows of 4 columns (f32) or 4 bf16
  int vec16_ok;             // 16-byte aligned rows of 8 bf16 columns
  int32_t* dev_status;
  int splits;               // split-K factor (1 = none)
  float* partial;           // split-K partial sums [splits][M][N] (raw, no alpha)
};

// One GEMM request (host side).
struct GemmCall {
  int fmt;
  int64_t M, N, K;
  const uint8_t* a_codes;   // [M][K/2]
  const uint8_t* a_scales;
  const float* a_tensor_scale;
  const uint8_t* b_codes;   // [N][K/2]
  const uint8_t* b_scales;
  const float* b_tensor_scale;
  const void* lr_a;         // bf16 [M][lr_k] or NULL
  const void* lr_b;         // bf16 [N][lr_k] or NULL
  int64_t lr_k;             // multiple of 64 (0 = none)
  void* C;                  // output (NULL allowed with splits > 1 to keep partials only)
  int c_dtype;
  int64_t ldc;
  int bn;                   // MMA N tile: 64, 128 or 256 (an unsplit 256 may run as the 256 x 192 wide tile)
  int splits;
  float* partial;
  int32_t* dev_status;
};

metis_status run_gemm_fp4(const GemmCall& g, cudaStream_t s);

// The split count run_gemm_fp4 uses for a requested one: at most one split
// per 256-element K tile, and the fewest splits of the same length (so
// every split owns at least one K tile).  Partial sums are laid out
// [split][M][N].
int gemm_effective_splits(int64_t K, int splits);

}  // namespace metis
