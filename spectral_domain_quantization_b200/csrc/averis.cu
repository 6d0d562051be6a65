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

constexpr int kColsPerThread = 8;                     // one 16-byte bf16 load (two for f32)
constexpr int kColsPerBlock = 32 * kColsPerThread;    // a warp spans 256 columns
constexpr int kRowGroups = 8;                         // warps, interleaved over the rows
constexpr int kRowUnroll = 4;                         // rows whose loads are in flight together

// 8 consecutive elements of one row from column c (c + 8 <= n: vector loads).
MDEV void load8(const void* X, int dtype, int64_t idx, float* v) {
  if (dtype == METIS_BF16) {
    const uint4 u = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(X) + idx);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
    const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(X) + idx);
    const float4 b = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(X) + idx + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

// Block (column tile of 256, row chunk): warp w takes rows r0 + w, r0 + w + 8,
// ...; lane l takes columns tile*256 + 8 l .. + 7 (16-byte loads, a warp
// reads 512 contiguous bytes of a bf16 row), four rows' loads in flight at a
// time.  Per column: a float64 sum in row order within the warp, then the
// warps' sums in warp order; minimum and maximum.
__global__ void __launch_bounds__(32 * kRowGroups) colstats_kernel(const void* X, int dtype, int64_t m, int64_t n,
                                                                   int64_t ld, int64_t chunk_rows, double* psum,
                                                                   float* pmin, float* pmax) {
  __shared__ double ssum[kRowGroups][kColsPerBlock];
  __shared__ float smin[kRowGroups][kColsPerBlock], smax[kRowGroups][kColsPerBlock];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t c = static_cast<int64_t>(blockIdx.x) * kColsPerBlock + kColsPerThread * lane;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * chunk_rows;
  const int64_t r1 = imin64(m, r0 + chunk_rows);
  double sm[kColsPerThread];
  float mn[kColsPerThread], mx[kColsPerThread];
#pragma unroll
  for (int j = 0; j < kColsPerThread; ++j) {
    sm[j] = 0.0;
    mn[j] = INFINITY;
    mx[j] = -INFINITY;
  }
  const bool full = c + kColsPerThread <= n;
  if (c < n) {
    int64_t r = r0 + w;
    for (; r + (kRowUnroll - 1) * kRowGroups < r1; r += kRowUnroll * kRowGroups) {
      float v[kRowUnroll][kColsPerThread];
#pragma unroll
      for (int u = 0; u < kRowUnroll; ++u) {
        const int64_t idx = (r + u * kRowGroups) * ld + c;
        if (full) {
          load8(X, dtype, idx, v[u]);
        } else {
#pragma unroll
          for (int j = 0; j < kColsPerThread; ++j) v[u][j] = c + j < n ? load_elem(X, dtype, idx + j) : 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < kRowUnroll; ++u) {
#pragma unroll
        for (int j = 0; j < kColsPerThread; ++j) {
          sm[j] += v[u][j];
          mn[j] = fminf(mn[j], v[u][j]);
          mx[j] = fmaxf(mx[j], v[u][j]);
        }
      }
    }
    for (; r < r1; r += kRowGroups) {
      float v[kColsPerThread];
      const int64_t idx = r * ld + c;
      if (full) {
        load8(X, dtype, idx, v);
      } else {
#pragma unroll
        for (int j = 0; j < kColsPerThread; ++j) v[j] = c + j < n ? load_elem(X, dtype, idx + j) : 0.f;
      }
#pragma unroll
      for (int j = 0; j < kColsPerThread; ++j) {
        sm[j] += v[j];
        mn[j] = fminf(mn[j], v[j]);
        mx[j] = fmaxf(mx[j], v[j]);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < kColsPerThread; ++j) {
    ssum[w][kColsPerThread * lane + j] = sm[j];
    smin[w][kColsPerThread * lane + j] = mn[j];
    smax[w][kColsPerThread * lane + j] = mx[j];
  }
  __syncthreads();
  const int t = threadIdx.x;   // one column of the tile
  const int64_t col = static_cast<int64_t>(blockIdx.x) * kColsPerBlock + t;
  if (col < n) {
    double sum = 0.0;
    float lo = INFINITY, hi = -INFINITY;
    for (int g = 0; g < kRowGroups; ++g) {
      sum += ssum[g][t];
      lo = fminf(lo, smin[g][t]);
      hi = fmaxf(hi, smax[g][t]);
    }
    const int64_t o = static_cast<int64_t>(blockIdx.y) * n + col;
    psum[o] = sum;
    pmin[o] = lo;
    pmax[o] = hi;
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
  colstats_kernel<<<grid, 32 * kRowGroups, 0, s>>>(X, dtype, m, n, ld, chunk_rows, psum, pmin, pmax);
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
