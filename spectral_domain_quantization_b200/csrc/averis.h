// Interface of the Averis column statistics (averis.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace metis {

int64_t colstats_chunk_rows(int64_t m, int64_t n, int sms);
// mean[n] = column means (float32 of a float64 sum); *amax_bits = max |x - mean|
// over the matrix (float bits).  psum / pmin / pmax: ceil(m / chunk_rows) * n
// entries of scratch each.
// R = fl32(X - 1 mu^T) as float32 (m x n, row-major), without quantizing.
void launch_residual_tap(const void* X, int dtype, int64_t m, int64_t n, int64_t ld, const float* mu, float* R,
                         int num_sms, cudaStream_t s);
void launch_colstats(const void* X, int dtype, int64_t m, int64_t n, int64_t ld, int64_t chunk_rows, double* psum,
                     float* pmin, float* pmax, float* mean, unsigned* amax_bits, cudaStream_t s);

}  // namespace metis
