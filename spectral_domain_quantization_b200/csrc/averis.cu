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
#include "abi_common.h"
#include "common.cuh"
#include "averis.h"

namespace metis {

namespace {

constexpr int kColsPerThread = 8;                     // one 16-byte bf16 load (two for f32)
constexpr int kColsPerBlock = 32 * kColsPerThread;    // a warp spans 256 columns
constexpr int kRowGroups = 8;                         // warps, interleaved over the rows
constexpr int kRowUnroll = 2;                         // rows whose loads are in flight together

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
__global__ void __launch_bounds__(32 * kRowGroups, 3) colstats_kernel(const void* X, int dtype, int64_t m, int64_t n,
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

// The same statistics for a bf16 X streamed by TMA (more bytes in flight
// than register-staged loads allow): one producer warp feeds 64 x 64 tiles of
// a 64-column strip through a ring of shared-memory stages; consumer warp w
// takes tiles w, w + 8, ... of each (strip, run of row tiles) item.  Lane
// (c, r) reduces 8 columns (16-byte row reads, the 8 lanes of a row reading
// 128 contiguous bytes) over rows 16 r .. 16 r + 15 of each tile: float64
// sums in row order, then the 4 row lanes in a fixed order, and each warp
// writes one partial per column and item (chunk run * 8 + w).
constexpr int kStatTile = 64;
constexpr int kStatConsumers = 8;
constexpr int kStatStages = 12;           // 96 KB of stages: two CTAs per SM
static_assert((2 * kStatStages) % kStatConsumers == 0, "a stage's rounds must alternate between at most two warps");

struct StatArgs {
  int64_t m, n, strips, runs, run_tiles, ntiles;
};

__global__ void __launch_bounds__(32 * (kStatConsumers + 1), 2) colstats_tma_kernel(
    const StatArgs a, const __grid_constant__ CUtensorMap tmX, double* psum, float* pmin, float* pmax,
    int32_t* dev_status) {
  extern __shared__ __align__(1024) uint8_t st_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(st_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[kStatStages], empty[kStatStages];
  __shared__ int abort_sh;
  constexpr int kStageBytes = kStatTile * kStatTile * 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStatStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    abort_sh = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmX);
  }
  __syncthreads();
  volatile int* abort_flag = &abort_sh;
  const int64_t items = a.strips * a.runs;
  if (warp == kStatConsumers) {
    if (lane == 0) {
      int s = 0, issued = 0;    // stage, phase and count tracked as they go (no divisions per tile)
      uint32_t ph = 0;
      for (int64_t it = blockIdx.x; it < items && !*abort_flag; it += gridDim.x) {
        const int64_t run = it / a.strips, strip = it - run * a.strips;  // run-major: CTAs side by side read whole rows
        const int64_t g0 = run * a.run_tiles, g1 = imin64(a.ntiles, g0 + a.run_tiles);
        for (int64_t g = g0; g < g1; ++g) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) break;
          mbar_arrive_expect_tx(&full[s], kStageBytes);
          tma_load_2d(ring + s * kStageBytes, &tmX, &full[s], static_cast<int32_t>(strip * kStatTile),
                      static_cast<int32_t>(g * kStatTile));
          ++issued;
          if (++s == kStatStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (*abort_flag) {
        // let the copies in flight land before the CTA exits
        for (int k = 0; k < min(issued, kStatStages); ++k) {
          if (--s < 0) {
            s = kStatStages - 1;
            ph ^= 1u;
          }
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(&full[s], ph) && global_timer_ns() - t0 < 100000000ull) {
          }
        }
      }
    }
    return;
  }
  const int c = lane & 7, r = lane >> 3;   // 8 columns 8 c .. 8 c + 7, rows 16 r ..
  int qs = 0, turn = 0;   // tile q's stage, phase and consumer warp, tracked as q advances
  uint32_t qph = 0;
  for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
    const int64_t run = it / a.strips, strip = it - run * a.strips;  // run-major: CTAs side by side read whole rows
    const int64_t g0 = run * a.run_tiles, g1 = imin64(a.ntiles, g0 + a.run_tiles);
    double sm[8];
    float mn[8], mx[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      sm[j] = 0.0;
      mn[j] = INFINITY;
      mx[j] = -INFINITY;
    }
    for (int64_t g = g0; g < g1; ++g) {
      const int s = qs;
      const uint32_t sph = qph;
      const bool mine = turn == warp;
      if (++qs == kStatStages) {
        qs = 0;
        qph ^= 1u;
      }
      if (++turn == kStatConsumers) turn = 0;
      if (!mine) continue;
      // Stage s's rounds alternate between this warp and at most one other
      // (2 x the stage count is a multiple of the consumer warps), so the
      // round before this one may be the other warp's and its load may still
      // be in flight, when a parity wait on full[s] would pass a phase early.
      // Its consumption on empty[s] comes first: at once for the first round
      // and for a round this warp consumed itself.
      if (!mbar_wait(&empty[s], sph ^ 1u, abort_flag)) break;
      if (!mbar_wait(&full[s], sph, abort_flag)) break;
      const uint8_t* tile = ring + s * kStageBytes;
      const int nr = static_cast<int>(imin64(16, a.m - (g * kStatTile + 16 * r)));  // rows of this lane in X
#pragma unroll 4
      for (int i = 0; i < 16; ++i) {
        if (i < nr) {
          const uint4 w = *reinterpret_cast<const uint4*>(tile + (16 * r + i) * 128 + 16 * c);
          const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float lo = __uint_as_float(x[k] << 16), hi = __uint_as_float(x[k] & 0xFFFF0000u);
            sm[2 * k] += lo;
            sm[2 * k + 1] += hi;
            mn[2 * k] = fminf(mn[2 * k], lo);
            mx[2 * k] = fmaxf(mx[2 * k], lo);
            mn[2 * k + 1] = fminf(mn[2 * k + 1], hi);
            mx[2 * k + 1] = fmaxf(mx[2 * k + 1], hi);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);   // every value read from the stage has been used
    }
    // the four row lanes of each column group: r = 0 + 1, 2 + 3, then the pair sums
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int off = 8; off < 32; off <<= 1) {
        sm[j] += __shfl_xor_sync(0xFFFFFFFFu, sm[j], off);
        mn[j] = fminf(mn[j], __shfl_xor_sync(0xFFFFFFFFu, mn[j], off));
        mx[j] = fmaxf(mx[j], __shfl_xor_sync(0xFFFFFFFFu, mx[j], off));
      }
    }
    if (r == 0) {
      const int64_t chunk = run * kStatConsumers + warp;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t col = strip * kStatTile + 8 * c + j;
        if (col < a.n) {
          psum[chunk * a.n + col] = sm[j];
          pmin[chunk * a.n + col] = mn[j];
          pmax[chunk * a.n + col] = mx[j];
        }
      }
    }
  }
  if (threadIdx.x == 0 && *abort_flag) report(dev_status, METIS_DEV_TIMEOUT);
}

StatArgs stat_args(int64_t m, int64_t n, int sms) {
  StatArgs a{};
  a.m = m;
  a.n = n;
  a.strips = (n + kStatTile - 1) / kStatTile;
  a.ntiles = (m + kStatTile - 1) / kStatTile;
  int64_t runs = imax64(1, imin64(a.ntiles, (4 * static_cast<int64_t>(sms) + a.strips - 1) / a.strips));
  a.run_tiles = (a.ntiles + runs - 1) / runs;
  a.runs = (a.ntiles + a.run_tiles - 1) / a.run_tiles;
  return a;
}

bool colstats_tma_ok(const void* X, int dtype, int64_t n, int64_t ld) {
  return dtype == METIS_BF16 && (reinterpret_cast<uintptr_t>(X) & 15u) == 0 && (ld * 2) % 16 == 0 && n % 8 == 0;
}

// mu_j = fl32(sum_j / m); residual tensor max from the column extremes.
// A CTA takes 32 columns (a lane each, coalesced rows of the partials); its 8
// warps take every 8th chunk, and warp 0 adds the 8 warp sums in warp order
// (the sum is deterministic).
constexpr int kFinGroups = 8;
__global__ void __launch_bounds__(32 * kFinGroups) colstats_finalize_kernel(const double* psum, const float* pmin,
                                                                          const float* pmax, int nchunks, int64_t m,
                                                                          int64_t n, float* mean,
                                                                          unsigned* amax_bits) {
  __shared__ double ssum[kFinGroups][32];
  __shared__ float smin[kFinGroups][32], smax[kFinGroups][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t j = static_cast<int64_t>(blockIdx.x) * 32 + lane;
  double sm = 0.0;
  float mn = INFINITY, mx = -INFINITY;
  if (j < n) {
#pragma unroll 4
    for (int b = w; b < nchunks; b += kFinGroups) {
      sm += psum[static_cast<int64_t>(b) * n + j];
      mn = fminf(mn, pmin[static_cast<int64_t>(b) * n + j]);
      mx = fmaxf(mx, pmax[static_cast<int64_t>(b) * n + j]);
    }
  }
  ssum[w][lane] = sm;
  smin[w][lane] = mn;
  smax[w][lane] = mx;
  __syncthreads();
  if (w != 0) return;
  float local = 0.f;
  if (j < n) {
    double t = 0.0;
    float lo = INFINITY, hi = -INFINITY;
#pragma unroll
    for (int g = 0; g < kFinGroups; ++g) {
      t += ssum[g][lane];
      lo = fminf(lo, smin[g][lane]);
      hi = fmaxf(hi, smax[g][lane]);
    }
    const float mu = static_cast<float>(t / static_cast<double>(m));
    mean[j] = mu;
    local = fmaxf(__fsub_rn(hi, mu), -__fsub_rn(lo, mu));
  }
  for (int o = 16; o > 0; o >>= 1) local = fmaxf(local, __shfl_xor_sync(0xFFFFFFFFu, local, o));
  if (lane == 0) atomicMax(amax_bits, __float_as_uint(local));
}

}  // namespace

int64_t colstats_chunks(const void* X, int dtype, int64_t m, int64_t n, int64_t ld, int sms) {
  if (colstats_tma_ok(X, dtype, n, ld)) return stat_args(m, n, sms).runs * kStatConsumers;
  const int64_t rows = colstats_chunk_rows(m, n, sms);
  return (m + rows - 1) / rows;
}

int64_t colstats_chunk_rows(int64_t m, int64_t n, int sms) {
  // enough row chunks that (column tiles x chunks) covers the GPU about 4 times
  const int64_t tiles = (n + kColsPerBlock - 1) / kColsPerBlock;
  int64_t chunks = (4 * static_cast<int64_t>(sms) + tiles - 1) / tiles;
  if (chunks < 1) chunks = 1;
  int64_t rows = (m + chunks - 1) / chunks;
  if (rows < kRowGroups) rows = kRowGroups;
  return rows;
}

void launch_colstats(const void* X, int dtype, int64_t m, int64_t n, int64_t ld, int sms, double* psum,
                     float* pmin, float* pmax, float* mean, unsigned* amax_bits, int32_t* dev_status,
                     cudaStream_t s) {
  if (colstats_tma_ok(X, dtype, n, ld)) {
    const StatArgs a = stat_args(m, n, sms);
    CUtensorMap map;
    const uint64_t dims[2] = {static_cast<uint64_t>(n), static_cast<uint64_t>(m)};
    const uint64_t strides[1] = {static_cast<uint64_t>(ld) * 2};
    const uint32_t box[2] = {kStatTile, kStatTile};
    if (encode_tensor_map(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, dims, strides, box,
                          CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS) {
      fail(METIS_ERR_CUDA, "colstats tensor map");
      return;
    }
    const size_t smem = static_cast<size_t>(kStatStages) * kStatTile * kStatTile * 2 + 1024;
    if (!ensure_smem(reinterpret_cast<const void*>(colstats_tma_kernel), smem)) return;
    const int grid = static_cast<int>(imin64(a.strips * a.runs, 2 * static_cast<int64_t>(sms)));
    colstats_tma_kernel<<<grid, 32 * (kStatConsumers + 1), smem, s>>>(a, map, psum, pmin, pmax, dev_status);
    const int64_t nchunks = a.runs * kStatConsumers;
    cudaMemsetAsync(amax_bits, 0, sizeof(unsigned), s);
    colstats_finalize_kernel<<<static_cast<unsigned>((n + 31) / 32), 32 * kFinGroups, 0, s>>>(
        psum, pmin, pmax, static_cast<int>(nchunks), m, n, mean, amax_bits);
    return;
  }
  const int64_t chunk_rows = colstats_chunk_rows(m, n, sms);
  const int64_t nchunks = (m + chunk_rows - 1) / chunk_rows;
  const dim3 grid(static_cast<unsigned>((n + kColsPerBlock - 1) / kColsPerBlock), static_cast<unsigned>(nchunks));
  colstats_kernel<<<grid, 32 * kRowGroups, 0, s>>>(X, dtype, m, n, ld, chunk_rows, psum, pmin, pmax);
  cudaMemsetAsync(amax_bits, 0, sizeof(unsigned), s);
  colstats_finalize_kernel<<<static_cast<unsigned>((n + 31) / 32), 32 * kFinGroups, 0, s>>>(
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
