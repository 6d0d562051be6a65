// Interface of the Averis column statistics (averis.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace metis {

int64_t colstats_chunk_rows(int64_t m, int64_t n, int sms);
// Partial chunks of the column statistics: psum / pmin / pmax need
// colstats_chunks(...) * n entries of scratch each.
int64_t colstats_chunks(const void* X, int dtype, int64_t m, int64_t n, int64_t ld, int sms);
// mean[n] = column means (float32 of a float64 sum); *amax_bits = max |x - mean|
// over the matrix (float bits).
// R = fl32(X - 1 mu^T) as float32 (m x n, row-major), without quantizing.
void launch_residual_tap(const void* X, int dtype, int64_t m, int64_t n, int64_t ld, const float* mu, float* R,
                         int num_sms, cudaStream_t s);
void launch_colstats(const void* X, int dtype, int64_t m, int64_t n, int64_t ld, int sms, double* psum,
                     float* pmin, float* pmax, float* mean, unsigned* amax_bits, int32_t* dev_status,
                     cudaStream_t s);

}  // namespace metis
