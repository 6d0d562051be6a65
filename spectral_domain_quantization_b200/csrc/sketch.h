// Interface of the sketch generators and the row sampler (sketch.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace metis {

constexpr int kMaxSparseNnz = 16;

// Radix-select state: the threshold key found so far and how many keys equal
// to it remain to be taken.
struct SelectState {
  uint64_t prefix;
  unsigned need;
  unsigned pad;
};

// Omega^T (lp rows of stride ldo) bf16: Gaussian (Philox + Box-Muller in float64).
void launch_gaussian_omega(int64_t n, int l, int lp, uint64_t seed, __nv_bfloat16* omt, int64_t ldo,
                           cudaStream_t s);
// Omega^T (lp x n) bf16: nnz entries +-1 per input coordinate.
void launch_sparse_sign(int64_t n, int l, int lp, int nnz, uint64_t seed, __nv_bfloat16* omt, int64_t ldo,
                        int32_t* dev_status, cudaStream_t s);
// idx[count]: the rows with the smallest Philox keys, ascending.  hist: 65536
// unsigned of scratch.
void launch_sample_rows(int64_t m, int64_t count, uint64_t seed, SelectState* st, unsigned* hist, int32_t* idx,
                        int sms, cudaStream_t s);
// out[j] = A[idx[j]] (whole rows of lda elements of size elem).
void launch_gather_rows(const void* A, int64_t n, int64_t lda, size_t elem, const int32_t* idx, int64_t count,
                        void* out, cudaStream_t s);

}  // namespace metis
