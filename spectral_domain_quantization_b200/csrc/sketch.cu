// Random sketch matrices and seeded row sampling (device side).
//
// Source: "Metis: Training LLMs with FP4 Quantization" abstract and technical
// framework (the dominant subspace survives sparse random sampling and random
// projection); SII release section 2.4 item 1 (randomized dimension
// reduction).  The generator is Philox4x32-10 (Salmon, Moraes, Dror, Shaw,
// SC'11): ten rounds of two 32x32->64-bit multiplies, key advanced by the Weyl
// constants between rounds.  Stream layout: counter word 2 selects the use
// (1 Gaussian sketch, 2 sparse-sign sketch, 3 row-sampling keys).
//
// The sketch is written transposed, Omega^T (lp x n, bf16, rows l..lp-1 zero),
// which is the K-major operand layout the sketch GEMM wants.
#include "common.cuh"
#include "sketch.h"

namespace metis {

namespace {

constexpr uint32_t kStreamOmega = 1, kStreamSparse = 2, kStreamSample = 3;

MDEV uint4 philox(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

// One thread per (row i, column pair c): Box-Muller in float64, rounded to bf16.
__global__ void gaussian_omega_kernel(int64_t n, int l, uint64_t seed, __nv_bfloat16* omt, int64_t ldo) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int c = blockIdx.y;
  if (i >= n) return;
  const uint4 w = philox(make_uint4(static_cast<uint32_t>(c), static_cast<uint32_t>(i), kStreamOmega, 0u),
                         static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
  const double u1 = (static_cast<double>(w.x) + 1.0) * 2.3283064365386963e-10;  // 2^-32
  const double u2 = static_cast<double>(w.y) * 2.3283064365386963e-10;
  const double r = sqrt(-2.0 * log(u1));
  const double theta = (2.0 * 3.141592653589793) * u2;
  omt[static_cast<int64_t>(2 * c) * ldo + i] = __double2bfloat16(r * cos(theta));
  if (2 * c + 1 < l) omt[static_cast<int64_t>(2 * c + 1) * ldo + i] = __double2bfloat16(r * sin(theta));
}

// One thread per input coordinate i: nnz distinct columns with random signs.
__global__ void sparse_sign_kernel(int64_t n, int l, int nnz, uint64_t seed, __nv_bfloat16* omt, int64_t ldo,
                                   int32_t* dev_status) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (i >= n) return;
  int taken[kMaxSparseNnz];
  int count = 0;
  for (uint32_t t = 0; t < 64u && count < nnz; ++t) {
    const uint4 w = philox(make_uint4(t, static_cast<uint32_t>(i), kStreamSparse, 0u), static_cast<uint32_t>(seed),
                           static_cast<uint32_t>(seed >> 32));
    const uint32_t cand[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (count >= nnz) break;
      const int col = static_cast<int>((static_cast<uint64_t>(cand[2 * h]) * static_cast<uint64_t>(l)) >> 32);
      bool dup = false;
      for (int q = 0; q < count; ++q) dup |= taken[q] == col;
      if (dup) continue;
      taken[count++] = col;
      omt[static_cast<int64_t>(col) * ldo + i] = __float2bfloat16((cand[2 * h + 1] >> 31) ? -1.f : 1.f);
    }
  }
  if (count < nnz) report(dev_status, METIS_DEV_SAMPLING);
}

MDEV uint64_t row_key(int64_t r, uint64_t seed) {
  const uint4 w = philox(make_uint4(static_cast<uint32_t>(r), 0u, kStreamSample, 0u), static_cast<uint32_t>(seed),
                         static_cast<uint32_t>(seed >> 32));
  return (static_cast<uint64_t>(w.y) << 32) | w.x;
}

// Radix select, one 16-bit digit per pass (most significant first): histogram
// of the digit over the keys that share the prefix chosen so far.
__global__ void key_hist_kernel(int64_t m, uint64_t seed, const SelectState* st, int pass, unsigned* hist) {
  const int shift = 48 - 16 * pass;
  for (int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; r < m;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint64_t k = row_key(r, seed);
    const uint64_t hi_mask = pass == 0 ? 0ull : (~0ull << (64 - 16 * pass));
    if ((k & hi_mask) != st->prefix) continue;
    atomicAdd(&hist[(k >> shift) & 0xFFFFu], 1u);
  }
}

// Single CTA: find the digit where the running count reaches `need`.
__global__ void key_pick_kernel(SelectState* st, int pass, unsigned* hist) {
  __shared__ unsigned part[1024];
  const int t = threadIdx.x;  // 1024 threads x 64 bins
  unsigned s = 0;
  for (int b = 0; b < 64; ++b) s += hist[t * 64 + b];
  part[t] = s;
  __syncthreads();
  if (t == 0) {
    unsigned run = 0, need = st->need;
    int chunk = 1023;
    for (int c = 0; c < 1024; ++c) {
      if (run + part[c] >= need) {
        chunk = c;
        break;
      }
      run += part[c];
    }
    unsigned digit = chunk * 64 + 63;
    for (int b = 0; b < 64; ++b) {
      const unsigned h = hist[chunk * 64 + b];
      if (run + h >= need) {
        digit = chunk * 64 + b;
        break;
      }
      run += h;
    }
    const int shift = 48 - 16 * pass;
    st->prefix |= static_cast<uint64_t>(digit) << shift;
    st->need = need - run;  // keys equal to the final key still to take
  }
  __syncthreads();
  for (int b = 0; b < 64; ++b) hist[t * 64 + b] = 0u;  // ready for the next pass
}

// Single CTA: ascending compaction of the selected rows (key < T, or key == T
// among the first `need` such rows).
__global__ void key_compact_kernel(int64_t m, uint64_t seed, const SelectState* st, int32_t* idx) {
  __shared__ unsigned wsum_sel[32], wsum_eq[32];
  __shared__ unsigned carry_sel, carry_eq;
  const uint64_t T = st->prefix;
  const unsigned need_eq = st->need;
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  if (t == 0) {
    carry_sel = 0;
    carry_eq = 0;
  }
  __syncthreads();
  for (int64_t base = 0; base < m; base += blockDim.x) {
    const int64_t r = base + t;
    uint64_t k = ~0ull;
    if (r < m) k = row_key(r, seed);
    const unsigned eq = (r < m && k == T) ? 1u : 0u;
    // rank among equal keys (inclusive scan)
    unsigned x = eq;
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned y = __shfl_up_sync(0xFFFFFFFFu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum_eq[w] = x;
    __syncthreads();
    unsigned before_eq = carry_eq;
    for (int q = 0; q < w; ++q) before_eq += wsum_eq[q];
    const unsigned eq_rank = before_eq + x - eq;  // exclusive
    const unsigned sel = (r < m) && (k < T || (eq && eq_rank < need_eq)) ? 1u : 0u;
    unsigned y2 = sel;
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned z = __shfl_up_sync(0xFFFFFFFFu, y2, o);
      if (lane >= o) y2 += z;
    }
    if (lane == 31) wsum_sel[w] = y2;
    __syncthreads();
    unsigned before_sel = carry_sel;
    for (int q = 0; q < w; ++q) before_sel += wsum_sel[q];
    if (sel) idx[before_sel + y2 - 1] = static_cast<int32_t>(r);
    __syncthreads();
    if (t == blockDim.x - 1) {
      carry_sel = before_sel + y2;
      carry_eq = before_eq + x;
    }
    __syncthreads();
  }
}

__global__ void gather_rows_kernel(const uint8_t* A, int64_t row_bytes, int64_t lda_bytes, const int32_t* idx,
                                   int64_t s, uint8_t* out) {
  const int64_t j = blockIdx.x;
  if (j >= s) return;
  const uint4* src = reinterpret_cast<const uint4*>(A + static_cast<int64_t>(idx[j]) * lda_bytes);
  uint4* dst = reinterpret_cast<uint4*>(out + j * row_bytes);
  for (int64_t q = threadIdx.x; q < row_bytes / 16; q += blockDim.x) dst[q] = src[q];
}

__global__ void init_select_kernel(SelectState* st, unsigned need) {
  st->prefix = 0;
  st->need = need;
}

}  // namespace

void launch_gaussian_omega(int64_t n, int l, int lp, uint64_t seed, __nv_bfloat16* omt, int64_t ldo,
                           cudaStream_t s) {
  cudaMemsetAsync(omt, 0, static_cast<size_t>(lp) * ldo * 2, s);
  const dim3 grid(static_cast<unsigned>((n + 255) / 256), static_cast<unsigned>((l + 1) / 2));
  gaussian_omega_kernel<<<grid, 256, 0, s>>>(n, l, seed, omt, ldo);
}

void launch_sparse_sign(int64_t n, int l, int lp, int nnz, uint64_t seed, __nv_bfloat16* omt, int64_t ldo,
                        int32_t* dev_status, cudaStream_t s) {
  cudaMemsetAsync(omt, 0, static_cast<size_t>(lp) * ldo * 2, s);
  sparse_sign_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(n, l, nnz, seed, omt, ldo, dev_status);
}

void launch_sample_rows(int64_t m, int64_t count, uint64_t seed, SelectState* st, unsigned* hist, int32_t* idx,
                        int sms, cudaStream_t s) {
  cudaMemsetAsync(hist, 0, 65536 * sizeof(unsigned), s);
  init_select_kernel<<<1, 1, 0, s>>>(st, static_cast<unsigned>(count));
  int blocks = static_cast<int>((m + 255) / 256);
  if (blocks > sms * 8) blocks = sms * 8;
  for (int pass = 0; pass < 4; ++pass) {
    key_hist_kernel<<<blocks, 256, 0, s>>>(m, seed, st, pass, hist);
    key_pick_kernel<<<1, 1024, 0, s>>>(st, pass, hist);
  }
  key_compact_kernel<<<1, 1024, 0, s>>>(m, seed, st, idx);
}

void launch_gather_rows(const void* A, int64_t n, int64_t lda, size_t elem, const int32_t* idx, int64_t count,
                        void* out, cudaStream_t s) {
  (void)n;  // whole rows of lda elements are copied, so the pitch stays 16-byte aligned
  gather_rows_kernel<<<static_cast<unsigned>(count), 256, 0, s>>>(
      static_cast<const uint8_t*>(A), lda * static_cast<int64_t>(elem), lda * static_cast<int64_t>(elem), idx, count,
      static_cast<uint8_t*>(out));
}

}  // namespace metis
