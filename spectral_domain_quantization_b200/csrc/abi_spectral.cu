// C ABI: metis_spectral_scale (see include/metis.h) -- adaptive spectral
// learning: the gradient G of a split weight preconditioned along the
// weight's singular directions.
//
// Source: SII release on Metis, section 2.4 item 2 (the gradients along the
// mid and low singular-value directions are scaled up by an inverse
// normalisation, without amplifying noise); "Metis: Training Large Language
// Models with Advanced Low-Bit Quantization", abstract item (ii) (adaptive
// learning rates in the spectral domain).
//
// With lambda_i = min(S_1 / S_i, cap) (1 where S_i <= 0), a = sqrt(lambda) - 1
// and C = U^T G V (k x k):
//   G' = (I + U a U^T) G (I + V a V^T)
//      = G + U (a P2^T) + (P1 a + U a C a) V^T,   P1 = G V, P2 = G^T U,
// a rank-2k update of G.  Enqueued pipeline:
//   G -> bf16 hi / lo parts; U^T, V^T -> bf16 hi / lo rows     (this file)
//   P1 = G V, P2 = G^T U                                       skinny passes
//   C = U^T P1                                                 (this file)
//   u = [U | P1 a + U a C a], w = -[P2 a | V] as bf16 hi / lo  (this file)
//   G' = G - u w^T, float32                                    residual pass
#include "abi_common.h"
#include "abi_internal.h"
#include "common.cuh"
#include "residual_quant.h"
#include "skinny_gemm.h"

namespace metis {

namespace {

constexpr int kMaxK = 64;     // 2k columns of the update fit the residual pass's 128
constexpr int kUpdateCols = 128;

MDEV float gain_root_minus_one(const float* S, int j, float cap) {
  // a_j = sqrt(lambda_j) - 1, lambda_j = min(S_0 / S_j, cap), 1 where S_j <= 0
  const float s0 = S[0], sj = S[j];
  if (!(s0 > 0.f) || !(sj > 0.f)) return 0.f;
  const float lam = fminf(s0 / sj, cap);
  return sqrtf(lam) - 1.f;
}

__global__ void hilo_kernel(const float* __restrict__ X, int64_t rows, int64_t cols, int64_t ld,
                            __nv_bfloat16* __restrict__ hi, __nv_bfloat16* __restrict__ lo) {
  const int64_t count = rows * cols;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < count;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = e / cols, c = e - r * cols;
    const float x = X[r * ld + c];
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    hi[r * ld + c] = h;
    lo[r * ld + c] = __float2bfloat16_rn(__fsub_rn(x, __bfloat162float(h)));
  }
}

// X (rows x k, row-major) -> X^T as bf16 hi rows [0, k) and lo rows
// [kq, kq + k) of outT (row stride ldo); the padding rows stay zero.
__global__ void transpose_hilo_kernel(const float* __restrict__ X, int64_t rows, int k, int kq,
                                      __nv_bfloat16* __restrict__ outT, int64_t ldo) {
  const int64_t count = rows * k;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < count;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(e / rows);
    const int64_t r = e - static_cast<int64_t>(c) * rows;   // rows fastest: coalesced stores
    const float x = X[r * k + c];
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    outT[static_cast<int64_t>(c) * ldo + r] = h;
    outT[static_cast<int64_t>(kq + c) * ldo + r] = __float2bfloat16_rn(__fsub_rn(x, __bfloat162float(h)));
  }
}

// C[i][j] = sum_r U[r][i] P1[r][j] (k x k): a warp per entry, float64 sums
// in a fixed order (lane-strided rows, then the warp tree).
__global__ void core_product_kernel(const float* __restrict__ U, const float* __restrict__ P1, int64_t rows, int k,
                                    int kq, float* __restrict__ C) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= k * k) return;
  const int i = warp / k, j = warp - i * k;
  double s = 0.0;
  for (int64_t r = lane; r < rows; r += 32) s = fma(static_cast<double>(U[r * k + i]), P1[r * kq + j], s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  if (lane == 0) C[i * k + j] = static_cast<float>(s);
}

MDEV void store_hilo(__nv_bfloat16* hi, __nv_bfloat16* lo, int64_t idx, float v) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  hi[idx] = h;
  lo[idx] = __float2bfloat16_rn(__fsub_rn(v, __bfloat162float(h)));
}

// Operands of the update, kUpdateCols columns each (zero past 2k):
//   u[r] = [U[r] | P1[r] a + U[r] a C a]      (rows of G)
//   w[n] = [-P2[n] a | -V[n]]                 (columns of G)
__global__ void update_operands_kernel(const float* __restrict__ U, const float* __restrict__ P1,
                                       const float* __restrict__ V, const float* __restrict__ P2,
                                       const float* __restrict__ S, const float* __restrict__ C, int64_t K,
                                       int64_t N, int k, int kq, float cap, __nv_bfloat16* u_hi,
                                       __nv_bfloat16* u_lo, __nv_bfloat16* w_hi, __nv_bfloat16* w_lo) {
  __shared__ float a[kMaxK];
  __shared__ float M[kMaxK * kMaxK];    // a C a
  for (int j = threadIdx.x; j < k; j += blockDim.x) a[j] = gain_root_minus_one(S, j, cap);
  __syncthreads();
  for (int e = threadIdx.x; e < k * k; e += blockDim.x) {
    const int i = e / k, j = e - i * k;
    M[e] = a[i] * C[e] * a[j];
  }
  __syncthreads();
  const int64_t total = (K + N) * kUpdateCols;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = e / kUpdateCols;
    const int c = static_cast<int>(e - row * kUpdateCols);
    float v = 0.f;
    if (row < K) {
      const int64_t r = row;
      if (c < k) {
        v = U[r * k + c];
      } else if (c < 2 * k) {
        const int j = c - k;
        float y = P1[r * kq + j] * a[j];
        for (int i = 0; i < k; ++i) y = fmaf(U[r * k + i], M[i * k + j], y);
        v = y;
      }
      store_hilo(u_hi, u_lo, r * kUpdateCols + c, v);
    } else {
      const int64_t n = row - K;
      if (c < k)
        v = -P2[n * kq + c] * a[c];
      else if (c < 2 * k)
        v = -V[n * k + (c - k)];
      store_hilo(w_hi, w_lo, n * kUpdateCols + c, v);
    }
  }
}

unsigned grid_for(int64_t items, int threads) {
  int64_t b = (items + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 8;
  if (b > cap) b = cap;
  return static_cast<unsigned>(b < 1 ? 1 : b);
}

int64_t round_up64(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

struct ScaleBuffers {
  __nv_bfloat16 *g_hi, *g_lo, *ut, *vt;
  float *P1, *P2, *C;
  __nv_bfloat16 *u_hi, *u_lo, *w_hi, *w_lo;
};

ScaleBuffers carve_scale(int64_t K, int64_t N, int64_t ldg, int k, Carver& ws) {
  const int kq = static_cast<int>(round_up64(k, 16));
  ScaleBuffers b{};
  b.g_hi = ws.take<__nv_bfloat16>(static_cast<size_t>(K) * ldg);
  b.g_lo = ws.take<__nv_bfloat16>(static_cast<size_t>(K) * ldg);
  b.ut = ws.take<__nv_bfloat16>(static_cast<size_t>(2 * kq) * round_up64(K, 8));
  b.vt = ws.take<__nv_bfloat16>(static_cast<size_t>(2 * kq) * round_up64(N, 8));
  b.P1 = ws.take<float>(static_cast<size_t>(K) * kq);
  b.P2 = ws.take<float>(static_cast<size_t>(N) * kq);
  b.C = ws.take<float>(static_cast<size_t>(k) * k);
  b.u_hi = ws.take<__nv_bfloat16>(static_cast<size_t>(K) * kUpdateCols);
  b.u_lo = ws.take<__nv_bfloat16>(static_cast<size_t>(K) * kUpdateCols);
  b.w_hi = ws.take<__nv_bfloat16>(static_cast<size_t>(N) * kUpdateCols);
  b.w_lo = ws.take<__nv_bfloat16>(static_cast<size_t>(N) * kUpdateCols);
  return b;
}

}  // namespace

}  // namespace metis

using namespace metis;

extern "C" metis_status metis_spectral_scale(const float* G, int64_t K, int64_t N, int64_t ldg, const float* U,
                                             const float* S, const float* V, int32_t k, float cap, float* Gout,
                                             void* workspace, size_t* workspace_bytes, int32_t* dev_status,
                                             void* stream) {
  if (!workspace_bytes) return METIS_ERR_NULL;
  if (!G || !U || !S || !V || !Gout || !dev_status) return METIS_ERR_NULL;
  METIS_TRY(validate_dense(G, METIS_F32, K, N, ldg));
  if (k < 1 || k > kMaxK) return METIS_ERR_ARG;
  if (!(cap >= 1.f) || !(cap < 3.4e38f)) return METIS_ERR_ARG;
  if (K % 32 || N % 32 || K > INT32_MAX || N > INT32_MAX) return METIS_ERR_SHAPE;
  if (static_cast<int64_t>(k) > K || static_cast<int64_t>(k) > N) return METIS_ERR_SHAPE;
  if (!aligned16(Gout)) return METIS_ERR_ALIGN;
  size_t need = 0;
  {
    Carver c(nullptr);
    carve_scale(K, N, ldg, k, c);
    need = c.used;
  }
  if (!workspace) {
    *workspace_bytes = need;
    return METIS_OK;
  }
  if (*workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return METIS_ERR_WORKSPACE;
  if (!device_is_sm100()) return METIS_ERR_UNSUPPORTED;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sms = device_sm_count();
  Carver ws(workspace);
  const ScaleBuffers b = carve_scale(K, N, ldg, k, ws);
  const int kq = static_cast<int>(round_up64(k, 16));
  const int64_t ldk = round_up64(K, 8), ldn = round_up64(N, 8);
  METIS_TRY(step_status("spectral_scale entry"));

  hilo_kernel<<<grid_for(K * N, 256), 256, 0, s>>>(G, K, N, ldg, b.g_hi, b.g_lo);
  cudaMemsetAsync(b.ut, 0, static_cast<size_t>(2 * kq) * ldk * sizeof(__nv_bfloat16), s);
  cudaMemsetAsync(b.vt, 0, static_cast<size_t>(2 * kq) * ldn * sizeof(__nv_bfloat16), s);
  transpose_hilo_kernel<<<grid_for(K * k, 256), 256, 0, s>>>(U, K, k, kq, b.ut, ldk);
  transpose_hilo_kernel<<<grid_for(N * k, 256), 256, 0, s>>>(V, N, k, kq, b.vt, ldn);
  METIS_TRY(step_status("spectral_scale operands"));

  SkinnyCall c{};
  c.m = K;
  c.n = N;
  c.lda = ldg;
  c.A[0] = b.g_hi;
  c.A[1] = b.g_lo;
  c.aparts = 2;
  c.xparts = 2;
  c.lp = kq;
  c.dev_status = dev_status;
  c.mode = 0;  // P1 = G V
  c.Xt = b.vt;
  c.ldx = ldn;
  c.cs = skinny_cluster(K, N, sms);
  c.out = b.P1;
  METIS_TRY(run_skinny_gemm(c, s));
  c.mode = 1;  // P2 = G^T U
  c.Xt = b.ut;
  c.ldx = ldk;
  c.cs = skinny_cluster(N, K, sms);
  c.out = b.P2;
  METIS_TRY(run_skinny_gemm(c, s));

  core_product_kernel<<<(k * k * 32 + 255) / 256, 256, 0, s>>>(U, b.P1, K, k, kq, b.C);
  update_operands_kernel<<<grid_for((K + N) * kUpdateCols, 256), 256, 0, s>>>(
      U, b.P1, V, b.P2, S, b.C, K, N, k, kq, cap, b.u_hi, b.u_lo, b.w_hi, b.w_lo);
  METIS_TRY(step_status("spectral_scale update operands"));

  // G' = G - u w^T, written as float32 by the residual pass (no FP4 outputs)
  ResidualOperands ro{b.u_hi, b.u_lo, b.w_hi, b.w_lo};
  ResidualParams rp{};
  rp.A = G;
  rp.dtype = METIS_F32;
  rp.m = K;
  rp.n = N;
  rp.lda = ldg;
  rp.kp = kUpdateCols;
  rp.fmt = METIS_MXFP4;   // no tensor scale is read: only the float32 output is written
  rp.mode = 1;
  rp.r_tap = Gout;
  rp.dev_status = dev_status;
  METIS_TRY(run_residual_quant(rp, ro, s));
  return launch_status();
}
