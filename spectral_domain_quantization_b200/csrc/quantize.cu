// FP4 block quantizer (MXFP4 / NVFP4) for dense bf16 / f32 matrices.
//
// Source: SII release on Metis, section 2.3 / Fig. 3 (block-wise quantization,
// each block's scale set by its maximum) and the feature list (MXFP4, NVFP4);
// Averis paragraphs of the arXiv 2603.10444 retelling (the optional per-column
// subtraction quantizes the mean-free residual).
//
// HBM-bound: every element is read once (twice for NVFP4, whose tensor maximum
// needs a pre-pass) and written as half a byte plus 1/16 or 1/32 byte of
// scale.  Work unit = one thread per 64 consecutive elements along the block
// axis (4 NVFP4 blocks or 2 MXFP4 blocks), so each thread writes 32 bytes of
// codes and a 32- or 16-bit word of the tensor-core scale layout.
//  * blocks along columns (axis 1): a thread reads 64 contiguous elements.
//  * blocks along rows (axis 0): a thread owns two adjacent columns and reads
//    64 rows of them; a warp covers 64 columns, i.e. 128 contiguous bytes of
//    each bf16 row.
#include "fp4_block.cuh"
#include "kernels.h"

namespace metis {

namespace {

constexpr int kGroup = 64;  // elements per thread along the block axis

MDEV float ld1(const void* X, int dtype, int64_t idx) { return load_elem(X, dtype, idx); }

// 8 consecutive elements from a 16-byte aligned address.
MDEV void ld8(const void* X, int dtype, int64_t idx, float* out) {
  if (dtype == METIS_BF16) {
    const uint4 u = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(X) + idx);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      out[2 * i] = __uint_as_float(w[i] << 16);
      out[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
    const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(X) + idx);
    const float4 b = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(X) + idx + 4);
    out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
    out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
  }
}

// two adjacent elements (idx even-aligned)
MDEV void ld2(const void* X, int dtype, int64_t idx, float& a, float& b) {
  if (dtype == METIS_BF16) {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(reinterpret_cast<const __nv_bfloat16*>(X) + idx);
    a = __uint_as_float(u << 16);
    b = __uint_as_float(u & 0xFFFF0000u);
  } else {
    const float2 f = *reinterpret_cast<const float2*>(reinterpret_cast<const float*>(X) + idx);
    a = f.x;
    b = f.y;
  }
}

// Quantize `n` (32 or 64) values of one outer index starting at inner offset
// g*64, write codes / scales / partial sum.
template <int FMT>
MDEV void emit_group(const float* v, int n, int64_t o, int64_t g, const QuantParams& p, float s_t) {
  uint8_t* codes = p.codes + o * (p.inner / 2) + g * (kGroup / 2);
  const int64_t c0 = g * (FMT == METIS_NVFP4 ? 4 : 2);
  float dsum_total = 0.f;
  uint32_t sc = 0;
  if (FMT == METIS_NVFP4) {
    uint64_t pk[4];
    const int nb = n / 16;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      pk[b] = 0;
      if (b < nb) {
        float ds;
        const uint32_t code = quant_block_nv(v + 16 * b, s_t, pk[b], ds);
        sc |= code << (8 * b);
        dsum_total += ds;
        if (p.scales_linear) p.scales_linear[o * (p.inner / 16) + c0 + b] = static_cast<uint8_t>(code);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(codes);
    dst[0] = make_uint4(static_cast<uint32_t>(pk[0]), static_cast<uint32_t>(pk[0] >> 32),
                        static_cast<uint32_t>(pk[1]), static_cast<uint32_t>(pk[1] >> 32));
    if (nb > 2)
      dst[1] = make_uint4(static_cast<uint32_t>(pk[2]), static_cast<uint32_t>(pk[2] >> 32),
                          static_cast<uint32_t>(pk[3]), static_cast<uint32_t>(pk[3] >> 32));
    *reinterpret_cast<uint32_t*>(p.scales + tc_scale_offset(o, c0, p.scale_cols)) = sc;
  } else {
    uint64_t pk[4];
    const int nb = n / 32;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      pk[2 * b] = pk[2 * b + 1] = 0;
      if (b < nb) {
        float ds;
        const uint32_t code = quant_block_mx(v + 32 * b, pk + 2 * b, ds);
        sc |= code << (8 * b);
        dsum_total += ds;
        if (p.scales_linear) p.scales_linear[o * (p.inner / 32) + c0 + b] = static_cast<uint8_t>(code);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(codes);
    dst[0] = make_uint4(static_cast<uint32_t>(pk[0]), static_cast<uint32_t>(pk[0] >> 32),
                        static_cast<uint32_t>(pk[1]), static_cast<uint32_t>(pk[1] >> 32));
    if (nb > 1)
      dst[1] = make_uint4(static_cast<uint32_t>(pk[2]), static_cast<uint32_t>(pk[2] >> 32),
                          static_cast<uint32_t>(pk[3]), static_cast<uint32_t>(pk[3] >> 32));
    *reinterpret_cast<uint16_t*>(p.scales + tc_scale_offset(o, c0, p.scale_cols)) =
        static_cast<uint16_t>(sc);
  }
  if (p.partial_sums) p.partial_sums[o * p.ngroups + g] = dsum_total;
}

MDEV float tensor_scale_of(const QuantParams& p) {
  if (p.fmt != METIS_NVFP4) return 1.f;
  const float alpha = __uint_as_float(*p.amax_bits);
  return nv_tensor_scale(alpha);
}

// blocks along columns: thread -> (row o, group g)
template <int FMT>
__global__ void __launch_bounds__(256) quantize_rows_kernel(QuantParams p) {
  const float s_t = tensor_scale_of(p);
  if (FMT == METIS_NVFP4 && blockIdx.x == 0 && threadIdx.x == 0 && p.tensor_scale) *p.tensor_scale = s_t;
  const int64_t total = p.outer * p.ngroups;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t o = t / p.ngroups;
    const int64_t g = t - o * p.ngroups;
    const int64_t i0 = g * kGroup;
    const int n = static_cast<int>(imin64(kGroup, p.inner - i0));
    float v[kGroup];
    const int64_t base = o * p.ld + i0;
#pragma unroll
    for (int j = 0; j < kGroup / 8; ++j) {
      if (8 * j < n) ld8(p.X, p.dtype, base + 8 * j, v + 8 * j);
    }
    if (p.sub) {
#pragma unroll
      for (int j = 0; j < kGroup; ++j)
        if (j < n) v[j] = __fsub_rn(v[j], p.sub[i0 + j]);
    }
    if (p.r_tap) {
#pragma unroll
      for (int j = 0; j < kGroup; ++j)
        if (j < n) p.r_tap[o * p.tap_ld + i0 + j] = v[j];
    }
    emit_group<FMT>(v, n, o, g, p, s_t);
  }
}

// blocks along rows: thread -> (column pair, group g of 64 rows)
template <int FMT>
__global__ void __launch_bounds__(256) quantize_cols_kernel(QuantParams p) {
  const float s_t = tensor_scale_of(p);
  if (FMT == METIS_NVFP4 && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0 &&
      threadIdx.y == 0 && p.tensor_scale)
    *p.tensor_scale = s_t;
  // p.outer = columns of X, p.inner = rows of X
  const int64_t c = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 2;
  const int64_t g = static_cast<int64_t>(blockIdx.y) * blockDim.y + threadIdx.y;
  if (c >= p.outer || g >= p.ngroups) return;
  const int64_t r0 = g * kGroup;
  const int n = static_cast<int>(imin64(kGroup, p.inner - r0));
  const bool two = c + 1 < p.outer;
  float va[kGroup], vb[kGroup];
  const float sa = p.sub ? p.sub[c] : 0.f;
  const float sb = (p.sub && two) ? p.sub[c + 1] : 0.f;
#pragma unroll
  for (int j = 0; j < kGroup; ++j) {
    if (j < n) {
      const int64_t idx = (r0 + j) * p.ld + c;
      if (two) {
        ld2(p.X, p.dtype, idx, va[j], vb[j]);
      } else {
        va[j] = ld1(p.X, p.dtype, idx);
        vb[j] = 0.f;
      }
      if (p.sub) {
        va[j] = __fsub_rn(va[j], sa);
        vb[j] = __fsub_rn(vb[j], sb);
      }
    }
  }
  if (p.r_tap) {
#pragma unroll
    for (int j = 0; j < kGroup; ++j) {
      if (j < n) {
        p.r_tap[(r0 + j) * p.tap_ld + c] = va[j];
        if (two) p.r_tap[(r0 + j) * p.tap_ld + c + 1] = vb[j];
      }
    }
  }
  emit_group<FMT>(va, n, c, g, p, s_t);
  if (two) emit_group<FMT>(vb, n, c + 1, g, p, s_t);
}

// max |x - sub| over the matrix into *out_bits (float bits, atomicMax).
__global__ void __launch_bounds__(256) amax_kernel(const void* X, int dtype, int64_t rows, int64_t cols,
                                                   int64_t ld, const float* sub, unsigned* out_bits) {
  float m = 0.f;
  const int64_t total = rows * cols;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t * 8 < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e = t * 8;
    const int64_t r = e / cols;
    const int64_t c = e - r * cols;
    float v[8];
    if (c + 8 <= cols && (cols % 8) == 0) {
      ld8(X, dtype, r * ld + c, v);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float x = sub ? __fsub_rn(v[j], sub[c + j]) : v[j];
        m = fmaxf(m, fabsf(x));
      }
    } else {
      for (int j = 0; j < 8 && e + j < total; ++j) {
        const int64_t rr = (e + j) / cols, cc = (e + j) - rr * cols;
        float x = load_elem(X, dtype, rr * ld + cc);
        if (sub) x = __fsub_rn(x, sub[cc]);
        m = fmaxf(m, fabsf(x));
      }
    }
  }
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
  __shared__ float wm[8];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.f;
    for (int i = 0; i < (blockDim.x >> 5); ++i) b = fmaxf(b, wm[i]);
    atomicMax(out_bits, __float_as_uint(b));
  }
}

__global__ void inner_sum_kernel(const float* partial, int64_t outer, int64_t ngroups, float* out) {
  const int64_t o = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (o >= outer) return;
  float s = 0.f;
  for (int64_t g = 0; g < ngroups; ++g) s += partial[o * ngroups + g];
  out[o] = s;
}

}  // namespace

int64_t quant_groups(int64_t inner) { return (inner + kGroup - 1) / kGroup; }

void launch_amax(const void* X, int dtype, int64_t rows, int64_t cols, int64_t ld, const float* sub,
                 unsigned* out_bits, int num_sms, cudaStream_t s) {
  const int64_t work = (rows * cols + 7) / 8;
  int blocks = static_cast<int>(imin64((work + 255) / 256, static_cast<int64_t>(num_sms) * 8));
  if (blocks < 1) blocks = 1;
  amax_kernel<<<blocks, 256, 0, s>>>(X, dtype, rows, cols, ld, sub, out_bits);
}

void launch_quantize(const QuantParams& p, int axis, int num_sms, cudaStream_t s) {
  if (axis == 1) {
    const int64_t total = p.outer * p.ngroups;
    int blocks = static_cast<int>(imin64((total + 255) / 256, static_cast<int64_t>(num_sms) * 16));
    if (blocks < 1) blocks = 1;
    if (p.fmt == METIS_NVFP4)
      quantize_rows_kernel<METIS_NVFP4><<<blocks, 256, 0, s>>>(p);
    else
      quantize_rows_kernel<METIS_MXFP4><<<blocks, 256, 0, s>>>(p);
  } else {
    const dim3 block(64, 4);
    const dim3 grid(static_cast<unsigned>((p.outer + 127) / 128),
                    static_cast<unsigned>((p.ngroups + 3) / 4));
    if (p.fmt == METIS_NVFP4)
      quantize_cols_kernel<METIS_NVFP4><<<grid, block, 0, s>>>(p);
    else
      quantize_cols_kernel<METIS_MXFP4><<<grid, block, 0, s>>>(p);
  }
  if (p.partial_sums && p.inner_sum) {
    inner_sum_kernel<<<static_cast<unsigned>((p.outer + 255) / 256), 256, 0, s>>>(
        p.partial_sums, p.outer, p.ngroups, p.inner_sum);
  }
}

}  // namespace metis
