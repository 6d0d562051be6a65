// Averis mean/residual split: column mean over all rows, mean-free residual.
//
// Source: retelling of arXiv 2603.10444 (mean bias in FP4 LLM training),
// Averis paragraphs: compute the mean over all rows of the activation matrix
// (one value per column), subtract it from every row by broadcasting, and
// quantize the mean vector and the residual separately; the backward pass
// splits the output gradient the same way.  The cost is two mean vectors and
// two subtractions.
//
// Pass 1 (this file): per column j, sum (float64), minimum and maximum over
// the rows, in fixed-order partial blocks -> mu_j = fl32(sum / m).  The NVFP4
// tensor maximum of the residual follows exactly from the column extremes:
// rounding is monotonic, so max_i |fl32(x_ij - mu_j)| is the larger of
// fl32(max_i x_ij - mu_j) and -fl32(min_i x_ij - mu_j).
// Pass 2 is the FP4 quantizer with the per-column subtraction (quantize.cu),
// once per requested block axis.
#include "common.cuh"
#include "averis.h"

namespace metis {

namespace {

constexpr int kColsPerBlock = 64;   // 32 threads x 2 columns
constexpr int kRowGroups = 8;       // threads per column pair

// Block (col tile, row chunk): 32 x 8 threads; thread (x, y) owns columns
// c = tile*64 + 2x, 2x+1 and rows r0 + y, r0 + y + 8, ...
__global__ void colstats_kernel(const void* X, int dtype, int64_t m, int64_t n, int64_t ld, int64_t chunk_rows,
                                double* psum, float* pmin, float* pmax) {
  __shared__ double ssum[kRowGroups][kColsPerBlock];
  __shared__ float smin[kRowGroups][kColsPerBlock], smax[kRowGroups][kColsPerBlock];
  const int x = threadIdx.x, y = threadIdx.y;
  const int64_t c = static_cast<int64_t>(blockIdx.x) * kColsPerBlock + 2 * x;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * chunk_rows;
  const int64_t r1 = imin64(m, r0 + chunk_rows);
  double s0 = 0.0, s1 = 0.0;
  float mn0 = INFINITY, mn1 = INFINITY, mx0 = -INFINITY, mx1 = -INFINITY;
  if (c < n) {
    const bool two = c + 1 < n;
    for (int64_t r = r0 + y; r < r1; r += kRowGroups) {
      float a, b = 0.f;
      const int64_t idx = r * ld + c;
      if (two) {
        if (dtype == METIS_BF16) {
          const uint32_t u = *reinterpret_cast<const uint32_t*>(reinterpret_cast<const __nv_bfloat16*>(X) + idx);
          a = __uint_as_float(u << 16);
          b = __uint_as_float(u & 0xFFFF0000u);
        } else {
          const float2 f = *reinterpret_cast<const float2*>(reinterpret_cast<const float*>(X) + idx);
          a = f.x;
          b = f.y;
        }
      } else {
        a = load_elem(X, dtype, idx);
      }
      s0 += a;
      mn0 = fminf(mn0, a);
      mx0 = fmaxf(mx0, a);
      if (two) {
        s1 += b;
        mn1 = fminf(mn1, b);
        mx1 = fmaxf(mx1, b);
      }
    }
  }
  ssum[y][2 * x] = s0;
  ssum[y][2 * x + 1] = s1;
  smin[y][2 * x] = mn0;
  smin[y][2 * x + 1] = mn1;
  smax[y][2 * x] = mx0;
  smax[y][2 * x + 1] = mx1;
  __syncthreads();
  const int t = y * 32 + x;
  if (t < kColsPerBlock) {
    const int64_t col = static_cast<int64_t>(blockIdx.x) * kColsPerBlock + t;
    if (col < n) {
      double s = 0.0;
      float mn = INFINITY, mx = -INFINITY;
      for (int g = 0; g < kRowGroups; ++g) {
        s += ssum[g][t];
        mn = fminf(mn, smin[g][t]);
        mx = fmaxf(mx, smax[g][t]);
      }
      const int64_t o = static_cast<int64_t>(blockIdx.y) * n + col;
      psum[o] = s;
      pmin[o] = mn;
      pmax[o] = mx;
    }
  }
}

// mu_j = fl32(sum_j / m); residual tensor max from the column extremes.
__global__ void colstats_finalize_kernel(const double* psum, const float* pmin, const float* pmax, int nchunks,
                                         int64_t m, int64_t n, float* mean, unsigned* amax_bits) {
  float local = 0.f;
  for (int64_t j = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; j < n;
       j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    double s = 0.0;
    float mn = INFINITY, mx = -INFINITY;
    for (int b = 0; b < nchunks; ++b) {
      s += psum[static_cast<int64_t>(b) * n + j];
      mn = fminf(mn, pmin[static_cast<int64_t>(b) * n + j]);
      mx = fmaxf(mx, pmax[static_cast<int64_t>(b) * n + j]);
    }
    const float mu = static_cast<float>(s / static_cast<double>(m));
    mean[j] = mu;
    local = fmaxf(local, fmaxf(__fsub_rn(mx, mu), -__fsub_rn(mn, mu)));
  }
  for (int o = 16; o > 0; o >>= 1) local = fmaxf(local, __shfl_xor_sync(0xFFFFFFFFu, local, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(local));
}

}  // namespace

int64_t colstats_chunk_rows(int64_t m, int64_t n, int sms) {
  // enough row chunks that (column tiles x chunks) covers the GPU about 4 times
  const int64_t tiles = (n + kColsPerBlock - 1) / kColsPerBlock;
  int64_t chunks = (4 * static_cast<int64_t>(sms) + tiles - 1) / tiles;
  if (chunks < 1) chunks = 1;
  int64_t rows = (m + chunks - 1) / chunks;
  if (rows < kRowGroups) rows = kRowGroups;
  return rows;
}

void launch_colstats(const void* X, int dtype, int64_t m, int64_t n, int64_t ld, int64_t chunk_rows, double* psum,
                     float* pmin, float* pmax, float* mean, unsigned* amax_bits, cudaStream_t s) {
  const int64_t nchunks = (m + chunk_rows - 1) / chunk_rows;
  const dim3 grid(static_cast<unsigned>((n + kColsPerBlock - 1) / kColsPerBlock), static_cast<unsigned>(nchunks));
  colstats_kernel<<<grid, dim3(32, kRowGroups), 0, s>>>(X, dtype, m, n, ld, chunk_rows, psum, pmin, pmax);
  cudaMemsetAsync(amax_bits, 0, sizeof(unsigned), s);
  colstats_finalize_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(
      psum, pmin, pmax, static_cast<int>(nchunks), m, n, mean, amax_bits);
}

// The float32 mean-free matrix alone: R[i][j] = fl32(x_ij - mu_j), the same
// float operation as the quantizers' tap (for callers that want the residual
// without its FP4 codes).  A grid-stride loop over elements, row-major.
__global__ void residual_tap_kernel(const void* X, int dtype, int64_t m, int64_t n, int64_t ld, const float* mu,
                                    float* R) {
  const int64_t total = m * n;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = e / n, j = e - i * n;
    const float x = dtype == METIS_BF16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(X)[i * ld + j])
                                        : reinterpret_cast<const float*>(X)[i * ld + j];
    R[e] = __fsub_rn(x, mu[j]);
  }
}

void launch_residual_tap(const void* X, int dtype, int64_t m, int64_t n, int64_t ld, const float* mu, float* R,
                         int num_sms, cudaStream_t s) {
  const int64_t total = m * n;
  int64_t blocks = (total + 255) / 256;
  if (blocks > static_cast<int64_t>(num_sms) * 8) blocks = static_cast<int64_t>(num_sms) * 8;
  if (blocks < 1) blocks = 1;
  residual_tap_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(X, dtype, m, n, ld, mu, R);
}

}  // namespace metis
