// FP4 block quantizer (MXFP4 / NVFP4) for dense bf16 / f32 matrices.
//
// Source: SII release on Metis, section 2.3 / Fig. 3 (block-wise quantization,
// each block's scale set by its maximum) and the feature list (MXFP4, NVFP4);
// Averis paragraphs of the arXiv 2603.10444 retelling (the optional per-column
// subtraction quantizes the mean-free residual).
//
// HBM-bound: every element is read once (twice for NVFP4, whose tensor maximum
// needs a pre-pass) and written as half a byte plus 1/16 or 1/32 byte of
// scale.  Blocks along columns: one thread per 64 consecutive elements (4
// NVFP4 blocks or 2 MXFP4 blocks), so each thread writes 32 bytes of codes
// and a 32- or 16-bit word of the tensor-core scale layout.
//  * blocks along columns (axis 1): a thread reads 64 contiguous elements.
//  * blocks along rows (axis 0): a CTA stages a 64 x 64 tile in shared
//    memory with coalesced row loads, then quantizes it column by column.
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

// Quantize `n` (32 or 64) values of one outer index starting at inner offset
// g*64, write codes / scales / (SUM) the group's partial sum.
template <int FMT, bool SUM>
MDEV void emit_group(const float* v, int n, int64_t o, int64_t g, const QuantParams& p, float s_t) {
  uint8_t* codes = p.codes + o * (p.inner / 2) + g * (kGroup / 2);
  const int64_t c0 = g * (FMT == METIS_NVFP4 ? 4 : 2);
  float dsum_total = 0.f;
  uint32_t sc = 0;
  uint64_t pk[4] = {0, 0, 0, 0};
  int nb;
  if (FMT == METIS_NVFP4) {
    nb = n / 16;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      if (b < nb) {
        float ds;
        const uint32_t code = quant_block_nv<SUM>(v + 16 * b, s_t, pk[b], ds);
        sc |= code << (8 * b);
        if (SUM) dsum_total += ds;
        if (p.scales_linear) p.scales_linear[o * (p.inner / 16) + c0 + b] = static_cast<uint8_t>(code);
      }
    }
    *reinterpret_cast<uint32_t*>(p.scales + tc_scale_offset(o, c0, p.scale_cols)) = sc;
    nb /= 2;  // 32-element halves written below
  } else {
    nb = n / 32;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      if (b < nb) {
        float ds;
        const uint32_t code = quant_block_mx<SUM>(v + 32 * b, pk + 2 * b, ds);
        sc |= code << (8 * b);
        if (SUM) dsum_total += ds;
        if (p.scales_linear) p.scales_linear[o * (p.inner / 32) + c0 + b] = static_cast<uint8_t>(code);
      }
    }
    *reinterpret_cast<uint16_t*>(p.scales + tc_scale_offset(o, c0, p.scale_cols)) = static_cast<uint16_t>(sc);
  }
  uint4* dst = reinterpret_cast<uint4*>(codes);
  dst[0] = make_uint4(static_cast<uint32_t>(pk[0]), static_cast<uint32_t>(pk[0] >> 32), static_cast<uint32_t>(pk[1]),
                      static_cast<uint32_t>(pk[1] >> 32));
  if (nb > 1)
    dst[1] = make_uint4(static_cast<uint32_t>(pk[2]), static_cast<uint32_t>(pk[2] >> 32),
                        static_cast<uint32_t>(pk[3]), static_cast<uint32_t>(pk[3] >> 32));
  if (SUM) p.partial_sums[o * p.ngroups + g] = dsum_total;
}

MDEV float tensor_scale_of(const QuantParams& p) {
  if (p.fmt != METIS_NVFP4) return 1.f;
  const float alpha = __uint_as_float(*p.amax_bits);
  return nv_tensor_scale(alpha);
}

// blocks along columns: thread -> (row o, group g)
template <int FMT, bool SUM>
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
    emit_group<FMT, SUM>(v, n, o, g, p, s_t);
  }
}

// blocks along columns: a grid-stride loop over 32-element units (2 NVFP4
// blocks or 1 MXFP4 block); the raw bytes of a thread's next unit are loaded
// before its current unit is quantized, so every thread keeps a load in
// flight while it computes.  With SUM (rows a multiple of 1024 elements, so a
// warp's 32 units always lie in one row) the warp adds its units' dequantized
// sums in a fixed tree order and lane 0 writes one partial per 1024 elements
// (partial_sums[o][u / 32], ngroups = inner / 1024).
template <int FMT, bool BF16, bool SUM, bool SUB>
__global__ void __launch_bounds__(256) quantize_rows_fast_kernel(QuantParams p) {
  constexpr int kU = 32;
  constexpr int kVec = BF16 ? 4 : 8;  // 16-byte words per unit
  __shared__ float enc_tab[128];
  const float s_t = tensor_scale_of(p);
  if (FMT == METIS_NVFP4 && blockIdx.x == 0 && threadIdx.x == 0 && p.tensor_scale) *p.tensor_scale = s_t;
  if (FMT == METIS_NVFP4) {
    nv_enc_table(s_t, enc_tab);
    __syncthreads();
  }
  const int64_t upr = p.inner / kU;  // inner is a multiple of 32
  const int64_t total = p.outer * upr;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const uint8_t* X = reinterpret_cast<const uint8_t*>(p.X);
  const int64_t esize = BF16 ? 2 : 4;
  // unit -> row: a 32-bit division while the unit count allows it
  const bool narrow = total < (int64_t{1} << 31);
  auto row_of = [&](int64_t unit) {
    return narrow ? static_cast<int64_t>(static_cast<uint32_t>(unit) / static_cast<uint32_t>(upr)) : unit / upr;
  };
  auto src = [&](int64_t unit) {
    const int64_t o = row_of(unit);
    return reinterpret_cast<const uint4*>(X + (o * p.ld + (unit - o * upr) * kU) * esize);
  };
  int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  // with the grid stride a multiple of the units per row, a thread keeps one
  // column unit for its whole loop, so its 32 column means are loaded once
  const bool fixed_u = SUB && stride % upr == 0;
  float subr[kU];
  if constexpr (SUB) {
    if (fixed_u && t < total) {
      const float* sp = p.sub + (t % upr) * kU;
      if ((reinterpret_cast<uintptr_t>(p.sub) & 15u) == 0) {
        const float4* s4 = reinterpret_cast<const float4*>(sp);
#pragma unroll
        for (int k = 0; k < kU / 4; ++k) {
          const float4 f = s4[k];
          subr[4 * k] = f.x;
          subr[4 * k + 1] = f.y;
          subr[4 * k + 2] = f.z;
          subr[4 * k + 3] = f.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < kU; ++j) subr[j] = sp[j];
      }
    }
  }
  uint4 cur[kVec], nxt[kVec];
  if (t < total) {
    const uint4* a = src(t);
#pragma unroll
    for (int k = 0; k < kVec; ++k) cur[k] = a[k];
  }
  for (; t < total; t += stride) {
    const int64_t tn = t + stride;
    if (tn < total) {
      const uint4* a = src(tn);
#pragma unroll
      for (int k = 0; k < kVec; ++k) nxt[k] = a[k];
    }
    const int64_t o = row_of(t), u = t - o * upr;
    float v[kU];
#pragma unroll
    for (int k = 0; k < kVec; ++k) {
      const uint32_t w[4] = {cur[k].x, cur[k].y, cur[k].z, cur[k].w};
      if (BF16) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[8 * k + 2 * i] = __uint_as_float(w[i] << 16);
          v[8 * k + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) v[4 * k + i] = __uint_as_float(w[i]);
      }
    }
    if constexpr (SUB) {
      if (fixed_u) {
#pragma unroll
        for (int j = 0; j < kU; ++j) v[j] = __fsub_rn(v[j], subr[j]);
      } else {
#pragma unroll
        for (int j = 0; j < kU; ++j) v[j] = __fsub_rn(v[j], p.sub[u * kU + j]);
      }
    }
    if (p.r_tap) {
      float* tp = p.r_tap + o * p.tap_ld + u * kU;
#pragma unroll
      for (int j = 0; j < kU; ++j) tp[j] = v[j];
    }
    uint4* dst = reinterpret_cast<uint4*>(p.codes + o * (p.inner / 2) + u * (kU / 2));
    float ds = 0.f;
    if (FMT == METIS_NVFP4) {
      uint64_t pk0, pk1;
      float ds0, ds1;
      const uint32_t c0 = quant_block_nv_tab<SUM>(v, s_t, enc_tab, pk0, ds0);
      const uint32_t c1 = quant_block_nv_tab<SUM>(v + 16, s_t, enc_tab, pk1, ds1);
      if (SUM) ds = ds0 + ds1;
      *dst = make_uint4(static_cast<uint32_t>(pk0), static_cast<uint32_t>(pk0 >> 32), static_cast<uint32_t>(pk1),
                        static_cast<uint32_t>(pk1 >> 32));
      *reinterpret_cast<uint16_t*>(p.scales + tc_scale_offset(o, 2 * u, p.scale_cols)) =
          static_cast<uint16_t>(c0 | (c1 << 8));
      if (p.scales_linear) {
        p.scales_linear[o * (p.inner / 16) + 2 * u] = static_cast<uint8_t>(c0);
        p.scales_linear[o * (p.inner / 16) + 2 * u + 1] = static_cast<uint8_t>(c1);
      }
    } else {
      uint64_t pk[2];
      const uint32_t c0 = quant_block_mx<SUM>(v, pk, ds);
      *dst = make_uint4(static_cast<uint32_t>(pk[0]), static_cast<uint32_t>(pk[0] >> 32),
                        static_cast<uint32_t>(pk[1]), static_cast<uint32_t>(pk[1] >> 32));
      p.scales[tc_scale_offset(o, u, p.scale_cols)] = static_cast<uint8_t>(c0);
      if (p.scales_linear) p.scales_linear[o * (p.inner / 32) + u] = static_cast<uint8_t>(c0);
    }
    if (SUM) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ds += __shfl_xor_sync(0xFFFFFFFFu, ds, off);
      if ((threadIdx.x & 31) == 0) p.partial_sums[o * (upr / 32) + u / 32] = ds;
    }
#pragma unroll
    for (int k = 0; k < kVec; ++k) cur[k] = nxt[k];
  }
}

// blocks along rows: CTA (x, y) takes the 64-column strip x of X and a run of
// consecutive 64-row groups [y G, y G + G).  Each group's 64 x 64 tile goes
// through shared memory (coalesced 16-byte row loads in, a column per
// thread group out); the next group's loads are issued into registers before
// the current tile is quantized, so loads stay in flight while the CTA
// computes.  Then each thread quantizes one block of one column (four
// threads, or two for MXFP4, cover a column's 64 rows, so their codes form
// one contiguous 32-byte segment).  With SUM the column's threads add their
// blocks' dequantized sums (shuffles, fixed order) and the first keeps a
// running sum over the run: one partial per column and run
// (partial_sums[o][y], ngroups = runs).
constexpr int kColTile = 64;

template <int FMT, bool SUM>
__global__ void __launch_bounds__(256) quantize_cols_kernel(QuantParams p, int64_t run) {
  constexpr int kBlk = FMT == METIS_NVFP4 ? 16 : 32;
  constexpr int kPerCol = kColTile / kBlk;  // threads per column
  constexpr int kSlots = kColTile * (kColTile / 8) / 256;  // 16-byte row segments per thread per tile
  __shared__ float tile[kColTile][kColTile + 1];
  __shared__ float enc_tab[128];
  const float s_t = tensor_scale_of(p);
  if (FMT == METIS_NVFP4 && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0 && p.tensor_scale)
    *p.tensor_scale = s_t;
  if (FMT == METIS_NVFP4) nv_enc_table(s_t, enc_tab);
  // p.outer = columns of X, p.inner = rows of X
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kColTile;
  const int nc = static_cast<int>(imin64(kColTile, p.outer - c0));
  const int64_t ngr = (p.inner + kColTile - 1) / kColTile;
  const int64_t g0 = static_cast<int64_t>(blockIdx.y) * run;
  const int64_t g1 = imin64(ngr, g0 + run);
  float raw[kSlots][8];
  auto fetch = [&](int64_t g) {
    const int64_t r0 = g * kColTile;
    const int nr = static_cast<int>(imin64(kColTile, p.inner - r0));
#pragma unroll
    for (int k = 0; k < kSlots; ++k) {
      const int e = threadIdx.x + 256 * k;
      const int r = e >> 3, q = (e & 7) * 8;
      if (r < nr && q + 8 <= nc) {
        ld8(p.X, p.dtype, (r0 + r) * p.ld + c0 + q, raw[k]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          raw[k][j] = (r < nr && q + j < nc) ? ld1(p.X, p.dtype, (r0 + r) * p.ld + c0 + q + j) : 0.f;
      }
    }
  };
  const int b = threadIdx.x % kPerCol, cc = threadIdx.x / kPerCol;  // this thread's block and column
  float subc[kSlots][8];  // the column means of this thread's row segments
#pragma unroll
  for (int k = 0; k < kSlots; ++k) {
    const int q = ((threadIdx.x + 256 * k) & 7) * 8;
#pragma unroll
    for (int j = 0; j < 8; ++j) subc[k][j] = (p.sub && q + j < nc) ? p.sub[c0 + q + j] : 0.f;
  }
  float colsum = 0.f;
  if (g0 < g1) fetch(g0);
  for (int64_t g = g0; g < g1; ++g) {
    const int64_t r0 = g * kColTile;
    const int nr = static_cast<int>(imin64(kColTile, p.inner - r0));
    __syncthreads();  // the previous tile has been read (and the encode table is ready)
#pragma unroll
    for (int k = 0; k < kSlots; ++k) {
      const int e = threadIdx.x + 256 * k;
      const int r = e >> 3, q = (e & 7) * 8;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float v = raw[k][j];
        if (p.sub && q + j < nc) v = __fsub_rn(v, subc[k][j]);
        tile[r][q + j] = v;
        if (p.r_tap && r < nr && q + j < nc) p.r_tap[(r0 + r) * p.tap_ld + c0 + q + j] = v;
      }
    }
    if (g + 1 < g1) fetch(g + 1);
    __syncthreads();
    const int nb = nr / kBlk;
    float ds = 0.f;
    if (threadIdx.x < kColTile * kPerCol && cc < nc && b < nb) {
      const int64_t o = c0 + cc;
      float v[kBlk];
#pragma unroll
      for (int i = 0; i < kBlk; ++i) v[i] = tile[b * kBlk + i][cc];
      uint8_t* dst = p.codes + o * (p.inner / 2) + (r0 + b * kBlk) / 2;
      const int64_t sc_col = (r0 + b * kBlk) / kBlk;
      uint32_t code;
      if (FMT == METIS_NVFP4) {
        uint64_t pk;
        code = quant_block_nv_tab<SUM>(v, s_t, enc_tab, pk, ds);
        *reinterpret_cast<uint2*>(dst) = make_uint2(static_cast<uint32_t>(pk), static_cast<uint32_t>(pk >> 32));
      } else {
        uint64_t pk[2];
        code = quant_block_mx<SUM>(v, pk, ds);
        *reinterpret_cast<uint4*>(dst) = make_uint4(static_cast<uint32_t>(pk[0]), static_cast<uint32_t>(pk[0] >> 32),
                                                    static_cast<uint32_t>(pk[1]), static_cast<uint32_t>(pk[1] >> 32));
      }
      p.scales[tc_scale_offset(o, sc_col, p.scale_cols)] = static_cast<uint8_t>(code);
      if (p.scales_linear) p.scales_linear[o * (p.inner / kBlk) + sc_col] = static_cast<uint8_t>(code);
    }
    if (SUM) {
      // the column's kPerCol threads are adjacent lanes: add their block sums
#pragma unroll
      for (int off = 1; off < kPerCol; off <<= 1) ds += __shfl_xor_sync(0xFFFFFFFFu, ds, off);
      colsum += ds;
    }
  }
  if (SUM && b == 0 && cc < nc) p.partial_sums[(c0 + cc) * p.ngroups + blockIdx.y] = colsum;
}

// max |x - sub| over the matrix into *out_bits (float bits, atomicMax).
__global__ void __launch_bounds__(256) amax_kernel(const void* X, int dtype, int64_t rows, int64_t cols,
                                                   int64_t ld, const float* sub, unsigned* out_bits) {
  float m = 0.f;
  const int64_t total = rows * cols;
  if (!sub && ld == cols && cols % 8 == 0) {
    // a dense matrix: one flat stream, two adjacent 8-element units per
    // thread and step (32 or 64 contiguous bytes), no index arithmetic
    const int64_t units = total / 8;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t t = 2 * (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x); t < units; t += 2 * stride) {
      float v0[8], v1[8];
      ld8(X, dtype, 8 * t, v0);
      if (t + 1 < units) {
        ld8(X, dtype, 8 * (t + 1), v1);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v1[j] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) m = fmaxf(m, fmaxf(fabsf(v0[j]), fabsf(v1[j])));
    }
  } else
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

// out[o] = sum of partial[o][0 .. ngroups): a warp per o, lanes strided over
// the groups (coalesced), then a fixed tree order.
__global__ void __launch_bounds__(256) inner_sum_kernel(const float* partial, int64_t outer, int64_t ngroups,
                                                        float* out) {
  const int64_t o = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (o >= outer) return;  // whole warps
  float s = 0.f;
  for (int64_t g = lane; g < ngroups; g += 32) s += partial[o * ngroups + g];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, off);
  if (lane == 0) out[o] = s;
}

}  // namespace

int64_t quant_groups(int64_t inner) { return (inner + kGroup - 1) / kGroup; }

void launch_amax(const void* X, int dtype, int64_t rows, int64_t cols, int64_t ld, const float* sub,
                 unsigned* out_bits, int num_sms, cudaStream_t s) {
  // no more CTAs than are resident at once: the grid-stride loop is
  // latency-bound, so a second wave would add its full length
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, amax_kernel, 256, 0) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const int64_t work = (rows * cols + 7) / 8;
  int blocks = static_cast<int>(imin64((work + 255) / 256, static_cast<int64_t>(num_sms) * per_sm));
  if (blocks < 1) blocks = 1;
  amax_kernel<<<blocks, 256, 0, s>>>(X, dtype, rows, cols, ld, sub, out_bits);
}

template <int FMT, bool SUM>
void launch_quantize_t(QuantParams& p, int axis, int num_sms, cudaStream_t s) {
  if (axis == 1 && (!SUM || p.inner % 1024 == 0)) {
    if (SUM) p.ngroups = p.inner / 1024;  // one partial per warp of units
    // two or more units per thread, so the prefetch overlaps; no more CTAs
    // than are resident at once (the grid-stride loop is latency-bound, so a
    // second wave would add its full length)
    const int64_t units = p.outer * (p.inner / 32);
    const bool bf = p.dtype == METIS_BF16, sub = p.sub != nullptr;
    const void* k = bf ? (sub ? reinterpret_cast<const void*>(quantize_rows_fast_kernel<FMT, true, SUM, true>)
                              : reinterpret_cast<const void*>(quantize_rows_fast_kernel<FMT, true, SUM, false>))
                       : (sub ? reinterpret_cast<const void*>(quantize_rows_fast_kernel<FMT, false, SUM, true>)
                              : reinterpret_cast<const void*>(quantize_rows_fast_kernel<FMT, false, SUM, false>));
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, 256, 0) != cudaSuccess || per_sm < 1) per_sm = 1;
    int blocks = static_cast<int>(imin64((units + 511) / 512, static_cast<int64_t>(num_sms) * per_sm));
    if (blocks < 1) blocks = 1;
    if (p.sub) {
      // a multiple of upr / gcd(upr, 256) CTAs makes the stride a multiple of
      // the units per row (each thread then keeps one column unit)
      int64_t a = p.inner / 32, b = 256;
      while (b) {
        const int64_t r = a % b;
        a = b;
        b = r;
      }
      const int64_t mult = (p.inner / 32) / a;
      if (mult <= 4 * static_cast<int64_t>(num_sms) * per_sm)
        blocks = static_cast<int>(imax64(mult, blocks / mult * mult));
    }
    if (bf && sub)
      quantize_rows_fast_kernel<FMT, true, SUM, true><<<blocks, 256, 0, s>>>(p);
    else if (bf)
      quantize_rows_fast_kernel<FMT, true, SUM, false><<<blocks, 256, 0, s>>>(p);
    else if (sub)
      quantize_rows_fast_kernel<FMT, false, SUM, true><<<blocks, 256, 0, s>>>(p);
    else
      quantize_rows_fast_kernel<FMT, false, SUM, false><<<blocks, 256, 0, s>>>(p);
  } else if (axis == 1) {
    const int64_t total = p.outer * p.ngroups;
    int blocks = static_cast<int>(imin64((total + 255) / 256, static_cast<int64_t>(num_sms) * 16));
    if (blocks < 1) blocks = 1;
    quantize_rows_kernel<FMT, SUM><<<blocks, 256, 0, s>>>(p);
  } else {
    // about one wave of CTAs (8 resident per SM), each over a run of row groups
    const int64_t strips = (p.outer + kColTile - 1) / kColTile;
    const int64_t ngr = (p.inner + kColTile - 1) / kColTile;
    int64_t runs = (static_cast<int64_t>(num_sms) * 8 + strips - 1) / strips;
    runs = runs < 1 ? 1 : (runs > ngr ? ngr : runs);
    const int64_t run = (ngr + runs - 1) / runs;
    runs = (ngr + run - 1) / run;
    if (SUM) p.ngroups = runs;   // one partial per column and run
    const dim3 grid(static_cast<unsigned>(strips), static_cast<unsigned>(runs));
    quantize_cols_kernel<FMT, SUM><<<grid, 256, 0, s>>>(p, run);
  }
}

void launch_quantize(const QuantParams& params, int axis, int num_sms, cudaStream_t s) {
  QuantParams p = params;  // the launcher may regroup the partial sums
  const bool sum = p.partial_sums != nullptr;
  if (quantize_tma_ok(p, axis, num_sms)) {
    if (sum) p.ngroups = quantize_tma_groups(p, axis, num_sms);
    launch_quantize_tma(p, axis, num_sms, nullptr, s);
    if (p.partial_sums && p.inner_sum)
      inner_sum_kernel<<<static_cast<unsigned>((p.outer * 32 + 255) / 256), 256, 0, s>>>(
          p.partial_sums, p.outer, p.ngroups, p.inner_sum);
    return;
  }
  if (p.fmt == METIS_NVFP4) {
    if (sum)
      launch_quantize_t<METIS_NVFP4, true>(p, axis, num_sms, s);
    else
      launch_quantize_t<METIS_NVFP4, false>(p, axis, num_sms, s);
  } else {
    if (sum)
      launch_quantize_t<METIS_MXFP4, true>(p, axis, num_sms, s);
    else
      launch_quantize_t<METIS_MXFP4, false>(p, axis, num_sms, s);
  }
  if (p.partial_sums && p.inner_sum) {
    inner_sum_kernel<<<static_cast<unsigned>((p.outer * 32 + 255) / 256), 256, 0, s>>>(
        p.partial_sums, p.outer, p.ngroups, p.inner_sum);
  }
}

}  // namespace metis
