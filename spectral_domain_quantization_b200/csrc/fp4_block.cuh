// One FP4 block: amax -> scale -> E2M1 codes, in the float32 op order of
// metis.h (MXFP4: OCP MX v1.0 scale rule; NVFP4: two-level scale).  Shared by
// the plain quantizer, the fused residual quantizer and the Averis quantizer.
#pragma once

#include "common.cuh"

namespace metis {

// NVFP4 tensor scale s_t = alpha / 2688 (1 when alpha == 0).
MDEV float nv_tensor_scale(float alpha) {
  return alpha == 0.f ? 1.f : __fdiv_rn(alpha, 2688.f);
}

// Sum of the 8 E2M1 values packed in w, as a multiple of 0.5 (exact), in
// integer arithmetic: a byte permute looks up twice each code's magnitude
// {0, 1, 2, 3, 4, 6, 8, 12} from an 8-byte table (selected by the code's 3
// magnitude bits), a second permute turns each sign bit into a +1 / -1 byte,
// and two signed 4-way byte dot products add the lot (twice the sum).
MDEV float e2m1_sum8(uint32_t w) {
  constexpr uint32_t kMagLo = 0x03020100u, kMagHi = 0x0C080604u, kSign = 0x0000FF01u;
  const uint32_t mlo = __byte_perm(kMagLo, kMagHi, w & 0x7777u);
  const uint32_t mhi = __byte_perm(kMagLo, kMagHi, (w >> 16) & 0x7777u);
  const uint32_t slo = __byte_perm(kSign, 0u, (w >> 3) & 0x1111u);
  const uint32_t shi = __byte_perm(kSign, 0u, (w >> 19) & 0x1111u);
  const int twice = __dp4a(static_cast<int>(mhi), static_cast<int>(shi),
                           __dp4a(static_cast<int>(mlo), static_cast<int>(slo), 0));
  return static_cast<float>(twice) * 0.5f;
}

// NVFP4 block of 16.  Returns the E4M3 scale code; writes 16 nibbles to
// `packed` (element i in bits 4i..4i+3) and, when SUM, the sum of the
// dequantized values to `dsum`.
template <bool SUM = false>
MDEV uint32_t quant_block_nv(const float* v, float s_t, uint64_t& packed, float& dsum) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(v[i]));
  const float t = __fdiv_rn(__fdiv_rn(a, s_t), 6.f);
  const uint32_t dc = e4m3_code(t);
  const float d = e4m3_value(dc);
  packed = 0;
  dsum = 0.f;
  if (d == 0.f) return dc;
  const float enc = __fdiv_rn(1.f, __fmul_rn(d, s_t));
  float q[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) q[i] = __fmul_rn(v[i], enc);
  const uint32_t w0 = e2m1_pack8(q), w1 = e2m1_pack8(q + 8);
  packed = static_cast<uint64_t>(w0) | (static_cast<uint64_t>(w1) << 32);
  if (SUM) {
    const float csum = e2m1_sum8(w0) + e2m1_sum8(w1);  // exact: 16 multiples of 0.5
    dsum = __fmul_rn(csum * d, s_t);                     // csum * d is exact in float32
  }
  return dc;
}

// The NVFP4 encode factors of one tensor: entry dc = 1 / (d(dc) s_t) for
// every E4M3 scale code dc (0 where d = 0), by the same float operations as
// quant_block_nv, so a block quantized through the table has the same codes.
// The calling CTA fills the 128 entries and synchronises before use.
MDEV void nv_enc_table(float s_t, float* tab) {
  for (int c = threadIdx.x; c < 128; c += blockDim.x) {
    const float d = e4m3_value(static_cast<uint32_t>(c));
    tab[c] = d == 0.f ? 0.f : __fdiv_rn(1.f, __fmul_rn(d, s_t));
  }
}

// quant_block_nv without the per-block reciprocal (taken from nv_enc_table);
// with SUM, the same dequantized sum as quant_block_nv<true>.
template <bool SUM = false>
MDEV uint32_t quant_block_nv_tab(const float* v, float s_t, const float* enc_tab, uint64_t& packed, float& dsum) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(v[i]));
  const float t = __fdiv_rn(__fdiv_rn(a, s_t), 6.f);
  const uint32_t dc = e4m3_code(t);
  packed = 0;
  dsum = 0.f;
  if (dc == 0u) return dc;  // d(0) = 0 and every other code has d > 0
  const float enc = enc_tab[dc];
  float q[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) q[i] = __fmul_rn(v[i], enc);
  const uint32_t w0 = e2m1_pack8(q), w1 = e2m1_pack8(q + 8);
  packed = static_cast<uint64_t>(w0) | (static_cast<uint64_t>(w1) << 32);
  if (SUM) {
    const float csum = e2m1_sum8(w0) + e2m1_sum8(w1);
    dsum = __fmul_rn(csum * e4m3_value(dc), s_t);
  }
  return dc;
}

MDEV uint32_t quant_block_nv_tab(const float* v, float s_t, const float* enc_tab, uint64_t& packed) {
  float unused;
  return quant_block_nv_tab<false>(v, s_t, enc_tab, packed, unused);
}

// MXFP4 block of 32.  Returns the E8M0 scale code; writes 32 nibbles to
// packed[0..1] and, when SUM, the sum of dequantized values to `dsum`.
template <bool SUM = false>
MDEV uint32_t quant_block_mx(const float* v, uint64_t* packed, float& dsum) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) a = fmaxf(a, fabsf(v[i]));
  packed[0] = packed[1] = 0;
  dsum = 0.f;
  if (a == 0.f) return 0u;
  int se = floor_log2(a) - 2;
  se = se < -127 ? -127 : (se > 127 ? 127 : se);
  const float inv = pow2f(-se);  // -se in [-125, 127]: a normal float
  float q[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) q[i] = __fmul_rn(v[i], inv);
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) w[j] = e2m1_pack8(q + 8 * j);
  packed[0] = static_cast<uint64_t>(w[0]) | (static_cast<uint64_t>(w[1]) << 32);
  packed[1] = static_cast<uint64_t>(w[2]) | (static_cast<uint64_t>(w[3]) << 32);
  if (SUM) {
    const float csum = (e2m1_sum8(w[0]) + e2m1_sum8(w[1])) + (e2m1_sum8(w[2]) + e2m1_sum8(w[3]));
    dsum = ldexpf(csum, se);
  }
  return static_cast<uint32_t>(se + 127);
}

}  // namespace metis
