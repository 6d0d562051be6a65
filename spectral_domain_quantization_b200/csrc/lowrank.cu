// Low-rank terms of the split-operand product, assembled into the bf16
// operands that the FP4 GEMM accumulates into its TMEM accumulator.
//
// Source: SII release on Metis, section 2.4 item 1 (the dominant rank-k part is
// quantized on its own and still enters the product); Averis paragraphs of
// the arXiv 2603.10444 retelling (mean and residual recombine in the output).
//
// For C = A B with A = R_A + F_A S_A P_A^T and B = R_B + P_B S_B F_B^T:
//   C = R_A R_B + T1 F_B^T + F_A T2,
//   T1 = (R_A P_B + F_A S_A (P_A^T P_B)) S_B     (M x kB)
//   T2 = S_A (P_A^T R_B)                          (kA x N)
// The GEMM accumulates alpha_main * (R_A R_B) with alpha_main the product of
// the residuals' tensor scales, so the low-rank operands are pre-divided by
// it.  Dequantized factors divided by their own tensor scale are exact in
// bf16 (<= 6 significant bits); fp32 T1/T2 enter as a bf16 hi/lo pair:
//   LA[m] = [hi(T1') | lo(T1') | F~_A | F~_A | 0...]
//   LB[n] = [F~_B    | F~_B    | hi(T2') | lo(T2') | 0...]
#include "abi_common.h"
#include "common.cuh"
#include "fp4_block.cuh"
#include "lowrank.h"

namespace metis {

namespace {

constexpr int kMaxLowRank = 128;   // k of one operand (checked by the ABI)

// Dequantized value of factor element (row i of `outer`, position l of
// `inner`) without the NVFP4 tensor scale.
MDEV float factor_value(const FactorView& f, int64_t i, int64_t l) {
  if (f.ones) return 1.f;
  const uint8_t byte = f.codes[i * (f.inner / 2) + (l >> 1)];
  const uint32_t code = (l & 1) ? (byte >> 4) : (byte & 15u);
  const int bs = f.fmt == METIS_MXFP4 ? 32 : 16;
  const uint8_t sc = f.scales[tc_scale_offset(i, l / bs, f.scale_cols)];
  const float s = f.fmt == METIS_MXFP4 ? ldexpf(1.f, static_cast<int>(sc) - 127) : e4m3_value(sc);
  return e2m1_value(code) * s;  // exact
}

MDEV float tscale(const FactorView& f) {
  return (f.ones || f.fmt != METIS_NVFP4 || !f.tensor_scale) ? 1.f : *f.tensor_scale;
}

// Cab[i][j] = sum_l P^_A[i][l] P^_B[j][l] (with tensor scales), a ka x kb
// product over the whole contraction.  Each CTA takes a run of positions,
// decodes both factors 64 positions at a time into shared memory (each
// value once, as float: exact) and accumulates 4 x 4 output tiles in
// registers; its partial goes to part[cta][i][j], and cab_reduce_kernel adds
// the partials in CTA order (deterministic) and applies the tensor scales.
constexpr int kCabStep = 64;     // positions decoded per round
constexpr int kCabThreads = 256;

__host__ __device__ inline int cab_pad(int k) { return (k + 3) / 4 * 4; }
__host__ __device__ inline int cab_stride(int k) { return cab_pad(k) + 4; }   // 16-byte rows, spread banks

__global__ void __launch_bounds__(kCabThreads) cab_part_kernel(FactorView pa, FactorView pb, int64_t K, int ka,
                                                               int kb, int64_t per_cta, float* part) {
  extern __shared__ float cab_sm[];
  const int sa = cab_stride(ka), sb = cab_stride(kb);
  float* A = cab_sm;                      // [kCabStep][sa]: A[l][i] = P^_A[i][l0 + l]
  float* B = A + kCabStep * sa;           // [kCabStep][sb]
  const int nib = cab_pad(ka) / 4, njb = cab_pad(kb) / 4, ntiles = nib * njb;
  const int64_t l0 = static_cast<int64_t>(blockIdx.x) * per_cta;
  const int64_t l1 = l0 + per_cta < K ? l0 + per_cta : K;
  constexpr int kMaxTiles = (kMaxLowRank / 4) * (kMaxLowRank / 4) / kCabThreads;
  float acc[kMaxTiles][4][4];
#pragma unroll
  for (int t = 0; t < kMaxTiles; ++t)
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int y = 0; y < 4; ++y) acc[t][x][y] = 0.f;
  for (int64_t base = l0; base < l1; base += kCabStep) {
    __syncthreads();   // the previous round's values are consumed
    for (int e = threadIdx.x; e < kCabStep * (cab_pad(ka) + cab_pad(kb)); e += kCabThreads) {
      const int l = e % kCabStep, r = e / kCabStep;
      const int64_t pos = base + l;
      const bool isa = r < cab_pad(ka);
      const int row = isa ? r : r - cab_pad(ka);
      const int lim = isa ? ka : kb;
      const float v = (row < lim && pos < l1) ? factor_value(isa ? pa : pb, row, pos) : 0.f;
      (isa ? A + l * sa : B + l * sb)[row] = v;
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < kMaxTiles; ++t) {
      const int tile = threadIdx.x + t * kCabThreads;
      if (tile < ntiles) {
        const int ib = tile % nib, jb = tile / nib;
#pragma unroll 4
        for (int l = 0; l < kCabStep; ++l) {
          const float4 x = *reinterpret_cast<const float4*>(A + l * sa + 4 * ib);
          const float4 y = *reinterpret_cast<const float4*>(B + l * sb + 4 * jb);
          const float xv[4] = {x.x, x.y, x.z, x.w}, yv[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
          for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int w = 0; w < 4; ++w) acc[t][u][w] = fmaf(xv[u], yv[w], acc[t][u][w]);
        }
      }
    }
  }
  float* out = part + static_cast<int64_t>(blockIdx.x) * ka * kb;
#pragma unroll
  for (int t = 0; t < kMaxTiles; ++t) {
    const int tile = threadIdx.x + t * kCabThreads;
    if (tile < ntiles) {
      const int ib = tile % nib, jb = tile / nib;
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int i = 4 * ib + u, j = 4 * jb + w;
          if (i < ka && j < kb) out[i * kb + j] = acc[t][u][w];
        }
    }
  }
}

__global__ void cab_reduce_kernel(FactorView pa, FactorView pb, int ka, int kb, int nparts, const float* part,
                                  float* cab) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= ka * kb) return;
  float s = 0.f;
  for (int c = 0; c < nparts; ++c) s += part[static_cast<int64_t>(c) * ka * kb + e];
  cab[e] = s * tscale(pa) * tscale(pb);
}

MDEV void split_hi_lo(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(__fsub_rn(x, __bfloat162float(hi)));
}

MDEV float alpha_main(const LowRankArgs& a) {
  float v = 1.f;
  if (a.ts_ra) v = __fmul_rn(v, *a.ts_ra);
  if (a.ts_rb) v = __fmul_rn(v, *a.ts_rb);
  return v;
}

// T1 element (m, j) before S_B: from T1 itself or from its split-K
// partials, summed in split order and scaled as the GEMM's own split-K
// reduction does (the same float operations, so the same value).
MDEV float t1_value(const LowRankArgs& a, int64_t m, int j) {
  if (a.t1part) {
    float s = 0.f;
    for (int k = 0; k < a.t1_splits; ++k) s += a.t1part[(k * a.M + m) * a.kb + j];
    float alpha = 1.f;
    if (a.t1_ts_a) alpha = __fmul_rn(alpha, *a.t1_ts_a);
    if (a.t1_ts_b) alpha = __fmul_rn(alpha, *a.t1_ts_b);
    return __fmul_rn(alpha, s);
  }
  return a.t1raw ? a.t1raw[m * a.t1_ld + j] : 0.f;
}

// One FP4 block (16 values NVFP4 / 32 MXFP4) of v, in place: v becomes
// code x block scale (exact in bf16), the tensor scale left out.
MDEV void requant_block(float* v, int fmt, float s_t) {
  float dsum;
  if (fmt == METIS_NVFP4) {
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = v[i];
    uint64_t packed;
    const float d = e4m3_value(quant_block_nv(x, s_t, packed, dsum));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = e2m1_value(static_cast<uint32_t>(packed >> (4 * i)) & 15u) * d;
  } else {
    float x[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) x[i] = v[i];
    uint64_t packed[2];
    const float d = ldexpf(1.f, static_cast<int>(quant_block_mx(x, packed, dsum)) - 127);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = e2m1_value(static_cast<uint32_t>(packed[i >> 4] >> (4 * (i & 15))) & 15u) * d;
  }
}

MDEV float requant_tensor_scale(const LowRankArgs& a, const unsigned* amax) {
  return a.fmt == METIS_NVFP4 ? nv_tensor_scale(__uint_as_float(*amax)) : 1.f;
}

MDEV void amax_update(unsigned* amax, float v) {
  unsigned u = __float_as_uint(fabsf(v));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) u = max(u, __shfl_xor_sync(0xffffffffu, u, o));
  if ((threadIdx.x & 31) == 0 && u) atomicMax(amax, u);
}

// T1 = (R_A P_B + F_A S_A (P_A^T P_B)) S_B in float32, element per thread,
// and (NVFP4) its absolute maximum.
__global__ void t1_form_kernel(LowRankArgs a) {
  const float s_fa = tscale(a.fa);
  const int64_t total = a.M * a.kb;
  const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t end = (total + step - 1) / step * step;   // whole warps take part in the reduction
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < end; t += step) {
    float v = 0.f;
    if (t < total) {
      const int64_t m = t / a.kb;
      const int j = static_cast<int>(t - m * a.kb);
      v = t1_value(a, m, j);
      if (a.ka > 0 && a.cab) {
        float acc = 0.f;
        for (int i = 0; i < a.ka; ++i) {
          const float sa = a.s_a ? a.s_a[i] : 1.f;
          acc += factor_value(a.fa, i, m) * s_fa * sa * a.cab[i * a.kb + j];
        }
        v += acc;
      }
      v = v * (a.s_b ? a.s_b[j] : 1.f);
      a.t1full[t] = v;
    }
    if (a.fmt == METIS_NVFP4) amax_update(a.amax1, v);
  }
}

// max |T2| with T2 = S_A (P_A^T R_B) (NVFP4).
__global__ void t2_amax_kernel(LowRankArgs a) {
  const int64_t total = static_cast<int64_t>(a.ka) * a.N;
  const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t end = (total + step - 1) / step * step;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < end; t += step) {
    float v = 0.f;
    if (t < total) {
      const int i = static_cast<int>(t / a.N);
      const int64_t n = t - static_cast<int64_t>(i) * a.N;
      v = a.t2raw[i * a.t2_ld + n] * (a.s_a ? a.s_a[i] : 1.f);
    }
    amax_update(a.amax2, v);
  }
}

// LA: a row per block iteration.  F_A's ka values at the row are decoded
// once into shared memory, T1's kb values (with the C_ab term) formed once,
// then the lr_k bf16 columns written a column per thread.
__global__ void build_la_kernel(LowRankArgs a) {
  __shared__ float row[kMaxLowRank];   // T1's row: re-quantized, or scaled for the hi / lo split
  __shared__ float far[kMaxLowRank];   // F_A at the row, without its tensor scale
  const float inv_alpha = 1.f / alpha_main(a);
  const float s_fb = tscale(a.fb);
  const float s_fa = tscale(a.fa);
  const float s_t1 = a.requant_t1 ? requant_tensor_scale(a, a.amax1) : 1.f;
  const float s_t2 = a.requant_t2 ? requant_tensor_scale(a, a.amax2) : 1.f;
  const int bs = a.fmt == METIS_MXFP4 ? 32 : 16;
  const int kbp = (a.kb + bs - 1) / bs * bs;
  for (int64_t m = blockIdx.x; m < a.M; m += gridDim.x) {
    for (int i = threadIdx.x; i < a.ka; i += blockDim.x) far[i] = factor_value(a.fa, i, m);
    // T1's row in blocks along kb (zero-padded), quantized and dequantized
    if (a.requant_t1)
      for (int j = threadIdx.x; j < kbp; j += blockDim.x) row[j] = j < a.kb ? a.t1full[m * a.kb + j] : 0.f;
    __syncthreads();
    if (a.requant_t1) {
      for (int b = threadIdx.x; b < kbp / bs; b += blockDim.x) requant_block(row + b * bs, a.fmt, s_t1);
    } else {
      for (int j = threadIdx.x; j < a.kb; j += blockDim.x) {
        float v = t1_value(a, m, j);
        if (a.ka > 0 && a.cab) {
          float acc = 0.f;
          for (int i = 0; i < a.ka; ++i) {
            const float sa = a.s_a ? a.s_a[i] : 1.f;
            acc += far[i] * s_fa * sa * a.cab[i * a.kb + j];
          }
          v += acc;
        }
        const float sb = a.s_b ? a.s_b[j] : 1.f;
        row[j] = v * sb * s_fb * inv_alpha;
      }
    }
    __syncthreads();
    for (int c = threadIdx.x; c < a.lr_k; c += blockDim.x) {
      __nv_bfloat16 out = __float2bfloat16_rn(0.f);
      if (c < 2 * a.kb) {
        const float v = row[c < a.kb ? c : c - a.kb];
        if (a.requant_t1) {
          // code x block scale in both chunks; the F_B side carries s_t1
          out = __float2bfloat16_rn(v);
        } else {
          __nv_bfloat16 hi, lo;
          split_hi_lo(v, hi, lo);
          out = c < a.kb ? hi : lo;
        }
      } else if (c < 2 * a.kb + 2 * a.ka) {
        const int cc = c - 2 * a.kb;
        const int i = cc % a.ka;
        if (a.requant_t2) {
          __nv_bfloat16 hi, lo;
          split_hi_lo(far[i] * s_fa * s_t2 * inv_alpha, hi, lo);
          out = cc < a.ka ? hi : lo;
        } else {
          out = __float2bfloat16_rn(far[i]);
        }
      }
      a.la[m * a.lr_k + c] = out;
    }
    __syncthreads();   // row and far are refilled next
  }
}

// LB: a row per block iteration, a column per thread.
__global__ void build_lb_kernel(LowRankArgs a) {
  __shared__ float col[kMaxLowRank];
  const float inv_alpha = 1.f / alpha_main(a);
  const float s_fa = tscale(a.fa);
  const float s_fb = tscale(a.fb);
  const float s_t1 = a.requant_t1 ? requant_tensor_scale(a, a.amax1) : 1.f;
  const float s_t2 = a.requant_t2 ? requant_tensor_scale(a, a.amax2) : 1.f;
  const int bs = a.fmt == METIS_MXFP4 ? 32 : 16;
  const int kap = (a.ka + bs - 1) / bs * bs;
  for (int64_t n = blockIdx.x; n < a.N; n += gridDim.x) {
    if (a.requant_t2) {
      // column n of T2 = S_A P_A^T R_B in blocks along ka (zero-padded)
      for (int i = threadIdx.x; i < kap; i += blockDim.x)
        col[i] = i < a.ka ? a.t2raw[i * a.t2_ld + n] * (a.s_a ? a.s_a[i] : 1.f) : 0.f;
      __syncthreads();
      for (int b = threadIdx.x; b < kap / bs; b += blockDim.x) requant_block(col + b * bs, a.fmt, s_t2);
      __syncthreads();
    }
    for (int c = threadIdx.x; c < a.lr_k; c += blockDim.x) {
      __nv_bfloat16 out = __float2bfloat16_rn(0.f);
      if (c < 2 * a.kb && a.requant_t1) {
        // F_B with its tensor scale and T1's, over the main alpha, as hi / lo
        const float w = factor_value(a.fb, c < a.kb ? c : c - a.kb, n) * s_fb * s_t1 * inv_alpha;
        __nv_bfloat16 hi, lo;
        split_hi_lo(w, hi, lo);
        out = c < a.kb ? hi : lo;
      } else if (c < 2 * a.kb) {
        out = __float2bfloat16_rn(factor_value(a.fb, c < a.kb ? c : c - a.kb, n));
      } else if (c < 2 * a.kb + 2 * a.ka && a.requant_t2) {
        // code x block scale of T2 in both chunks; the F_A side carries s_t2
        const int cc = c - 2 * a.kb;
        out = __float2bfloat16_rn(col[cc % a.ka]);
      } else if (c < 2 * a.kb + 2 * a.ka) {
        const int cc = c - 2 * a.kb;
        const int i = cc % a.ka;
        const float sa = a.s_a ? a.s_a[i] : 1.f;
        const float v = a.t2raw[i * a.t2_ld + n] * sa * s_fa * inv_alpha;
        __nv_bfloat16 hi, lo;
        split_hi_lo(v, hi, lo);
        out = cc < a.ka ? hi : lo;
      }
      a.lb[n * a.lr_k + c] = out;
    }
    if (a.requant_t2) __syncthreads();   // the column buffer is refilled next
  }
}

// Operands of the error-compensated residual: thread per (row, column c <
// kp) of [U rows | V rows]; column c < k holds hi / lo of deq(U_q)[row][c]
// (U's rows) or of fl32(deq(V_q)[row][c] S[c]) (V's rows), padding columns 0.
// deq includes the NVFP4 tensor scale.  The same [rows][kp] layout as the
// float32 factors' operands, which these replace.
__global__ void compensated_operands_kernel(FactorView fu, FactorView fv, int64_t m, int64_t n, int k,
                                            const float* S, int kp, __nv_bfloat16* u_hi, __nv_bfloat16* u_lo,
                                            __nv_bfloat16* w_hi, __nv_bfloat16* w_lo) {
  const float tu = tscale(fu), tv = tscale(fv);
  const int64_t total = (m + n) * kp;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = t / kp;
    const int c = static_cast<int>(t - row * kp);
    const bool isu = row < m;
    const int64_t r = isu ? row : row - m;
    float w = 0.f;
    if (c < k) w = isu ? __fmul_rn(factor_value(fu, c, r), tu) : __fmul_rn(__fmul_rn(factor_value(fv, c, r), tv), S[c]);
    const __nv_bfloat16 h = __float2bfloat16_rn(w);
    __nv_bfloat16* hi = isu ? u_hi : w_hi;
    __nv_bfloat16* lo = isu ? u_lo : w_lo;
    hi[r * kp + c] = h;
    lo[r * kp + c] = __float2bfloat16_rn(__fsub_rn(w, __bfloat162float(h)));
  }
}

int blocks_for(int64_t n, int sms) {
  int64_t b = (n + 255) / 256;
  if (b > sms * 8) b = sms * 8;
  return static_cast<int>(b < 1 ? 1 : b);
}

}  // namespace

int cab_parts(int64_t K, int sms) {
  const int64_t steps = (K + kCabStep - 1) / kCabStep;
  return static_cast<int>(steps < 2 * sms ? steps : 2 * sms);
}

bool launch_cab(const FactorView& pa, const FactorView& pb, int64_t K, int ka, int kb, float* part, float* cab,
                int sms, cudaStream_t s) {
  const int nparts = cab_parts(K, sms);
  const int64_t steps = (K + kCabStep - 1) / kCabStep;
  const int64_t per_cta = (steps + nparts - 1) / nparts * kCabStep;
  const int smem = kCabStep * (cab_stride(ka) + cab_stride(kb)) * static_cast<int>(sizeof(float));
  if (!ensure_smem(reinterpret_cast<const void*>(cab_part_kernel), static_cast<size_t>(smem))) return false;
  cab_part_kernel<<<nparts, kCabThreads, smem, s>>>(pa, pb, K, ka, kb, per_cta, part);
  cab_reduce_kernel<<<(ka * kb + 255) / 256, 256, 0, s>>>(pa, pb, ka, kb, nparts, part, cab);
  return true;
}

int row_blocks(int64_t rows, int sms) {
  const int64_t b = rows < sms * 16 ? rows : sms * 16;
  return static_cast<int>(b < 1 ? 1 : b);
}

void launch_build_lowrank(const LowRankArgs& a, int sms, cudaStream_t s) {
  const int threads = a.lr_k >= 128 ? 128 : 64;
  if (a.requant_t1 || a.requant_t2) {
    if (a.fmt == METIS_NVFP4) {
      if (a.requant_t1) cudaMemsetAsync(a.amax1, 0, sizeof(unsigned), s);
      if (a.requant_t2) cudaMemsetAsync(a.amax2, 0, sizeof(unsigned), s);
    }
    if (a.requant_t1) t1_form_kernel<<<blocks_for(a.M * a.kb, sms), 256, 0, s>>>(a);
    if (a.requant_t2 && a.fmt == METIS_NVFP4)
      t2_amax_kernel<<<blocks_for(static_cast<int64_t>(a.ka) * a.N, sms), 256, 0, s>>>(a);
  }
  build_la_kernel<<<row_blocks(a.M, sms), threads, 0, s>>>(a);
  build_lb_kernel<<<row_blocks(a.N, sms), threads, 0, s>>>(a);
}

void launch_compensated_operands(const FactorView& fu, const FactorView& fv, int64_t m, int64_t n, int k,
                                 const float* S, int kp, __nv_bfloat16* u_hi, __nv_bfloat16* u_lo,
                                 __nv_bfloat16* w_hi, __nv_bfloat16* w_lo, int sms, cudaStream_t s) {
  compensated_operands_kernel<<<blocks_for((m + n) * kp, sms), 256, 0, s>>>(fu, fv, m, n, k, S, kp, u_hi, u_lo, w_hi,
                                                                           w_lo);
}

}  // namespace metis
