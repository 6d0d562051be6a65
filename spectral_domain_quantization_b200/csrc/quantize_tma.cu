// FP4 block quantizer (MXFP4 / NVFP4) for bf16 matrices, fed by TMA: the
// streaming form of quantize.cu's kernels for the large activations and
// gradients (optional per-column subtraction and dequantized sums, as the
// Averis split needs them).
//
// Source: SII release on Metis, section 2.3 / Fig. 3 (block-wise quantization,
// each block's scale set by its maximum) and the feature list (MXFP4, NVFP4);
// Averis paragraphs of the arXiv 2603.10444 retelling (the per-column
// subtraction quantizes the mean-free residual).  The float arithmetic per
// block is quantize.cu's (fp4_block.cuh), so codes and scales are identical.
//
// HBM-bound: every element is read once and written as half a byte plus a
// scale byte per block.  Register-staged loads leave too few bytes in flight
// once the subtraction and the sums take registers, so here one producer warp
// streams 64 x 64 tiles of a 64-column strip (8 KB each; 64 x 128 for MXFP4
// along rows) through a ring of shared-memory stages with TMA, and 8
// consumer warps each quantize a whole tile: tile q goes to warp q mod 8 and
// stage q mod kStages.  A consumer hands its stage back only after every
// value it loaded from it has been used.
//  * blocks along columns (axis 1): a tile holds 64 rows x 2 units of 32
//    elements; lane (i, u) takes unit u of rows i, 16 + i, 32 + i, 48 + i.
//    The tile is 128-byte swizzled, so the 16-byte reads of a warp fall on
//    distinct bank groups.
//  * blocks along rows (axis 0): lane (b, g) takes block b of the 8 columns
//    8 g .. 8 g + 7 (NVFP4: 4 blocks of 16 rows; MXFP4: 2 blocks of 32 rows
//    over 128 columns); the 8 lanes of one row read 128 contiguous bytes.
// Work items are (strip, run of row tiles), numbered run-major so that the
// CTAs working at the same time cover whole rows; CTAs take items round-robin.
#include "abi_common.h"
#include "fp4_block.cuh"
#include "kernels.h"

namespace metis {

namespace {

constexpr int kTileRows = 64;
constexpr int kConsumers = 8;                   // consumer warps
constexpr int kQThreads = 32 * (kConsumers + 1);
// Blocks along columns: two CTAs per SM (96 KB rings); along rows the lanes
// hold more state, so one CTA per SM with the full register file (128 KB).
__host__ __device__ constexpr int ring_bytes(int axis) { return axis == 1 ? 96 * 1024 : 128 * 1024; }
__host__ __device__ constexpr int ctas_per_sm(int axis) { return axis == 1 ? 2 : 1; }

MDEV bool wait_until(uint64_t* bar, uint32_t parity, uint64_t ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > ns) return false;
  }
  return true;
}

struct TmaQuantArgs {
  QuantParams p;
  int64_t m, n;          // X rows, columns
  int64_t strips;        // column strips
  int64_t runs;          // row-tile runs per strip
  int64_t run_tiles;     // row tiles per run
  int64_t ntiles;        // row tiles (ceil(m / 64))
  int strip_cols;        // 64, or 128 for MXFP4 along rows
  int stages;
  int stage_bytes;
  int32_t* dev_status;
};

// Unpack 8 bf16 (one 16-byte word) to float.
MDEV void unpack8(const uint4& w, float* v) {
  const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(x[i] << 16);
    v[2 * i + 1] = __uint_as_float(x[i] & 0xFFFF0000u);
  }
}

template <int FMT, bool SUM, bool SUB, int AXIS>
__global__ void __launch_bounds__(kQThreads, ctas_per_sm(AXIS)) quantize_tma_kernel(const TmaQuantArgs a,
                                                                     const __grid_constant__ CUtensorMap tmX) {
  extern __shared__ __align__(1024) uint8_t qsm_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qsm_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[16], empty[16];
  __shared__ float enc_tab[128];
  __shared__ __align__(16) float wsub[kConsumers][2][32];   // each consumer warp's copy of its strip's column means
  __shared__ float wcol[kConsumers][2][8][32];  // blocks along rows: per lane, its 8 columns' mean and sum
  __shared__ int abort_sh;
  const QuantParams& p = a.p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.stages;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    abort_sh = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmX);
  }
  const float s_t = FMT == METIS_NVFP4 ? nv_tensor_scale(__uint_as_float(*p.amax_bits)) : 1.f;
  if (FMT == METIS_NVFP4) {
    nv_enc_table(s_t, enc_tab);
    if (blockIdx.x == 0 && threadIdx.x == 0 && p.tensor_scale) *p.tensor_scale = s_t;
  }
  __syncthreads();
  volatile int* abort_flag = &abort_sh;
  const int64_t items = a.strips * a.runs;

  if (warp == kConsumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0, issued = 0;    // stage, phase and count tracked as they go (no divisions per tile)
      uint32_t ph = 0;
      for (int64_t it = blockIdx.x; it < items && !*abort_flag; it += gridDim.x) {
        const int64_t run = it / a.strips, strip = it - run * a.strips;  // run-major: CTAs side by side read whole rows
        const int64_t g0 = run * a.run_tiles, g1 = imin64(a.ntiles, g0 + a.run_tiles);
        for (int64_t g = g0; g < g1; ++g) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) break;
          mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(a.stage_bytes));
          tma_load_2d(ring + s * a.stage_bytes, &tmX, &full[s], static_cast<int32_t>(strip * a.strip_cols),
                      static_cast<int32_t>(g * kTileRows));
          ++issued;
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (*abort_flag) {
        // let the copies in flight land before the CTA exits: the last
        // min(issued, S) stages, walking back from the next one
        for (int k = 0; k < min(issued, S); ++k) {
          if (--s < 0) {
            s = S - 1;
            ph ^= 1u;
          }
          wait_until(&full[s], ph, 100000000ull);
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int64_t outer_ld = p.inner / 2;   // code bytes per outer index
  // tile q's stage, phase and consumer warp, tracked as q advances
  int qs = 0, turn = 0;
  uint32_t qph = 0;
  for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
    const int64_t run = it / a.strips, strip = it - run * a.strips;  // run-major: CTAs side by side read whole rows
    const int64_t g0 = run * a.run_tiles, g1 = imin64(a.ntiles, g0 + a.run_tiles);
    const int64_t c0 = strip * a.strip_cols;  // first X column of the strip
    if (AXIS == 1) {
      // ---- blocks along columns: lane (i, u) -> unit u (32 columns) of
      //      rows i, 16 + i, 32 + i, 48 + i of each tile
      const int i = lane >> 1, u = lane & 1;
      const int64_t cu = c0 + 32 * u;          // the unit's first column
      const bool unit_ok = cu < a.n;
      if (SUB) {
        // this warp's copy of the strip's 64 means (read back as 16-byte vectors)
        __syncwarp();
#pragma unroll
        for (int h = 0; h < 2; ++h) wsub[warp][h][lane] = c0 + 32 * h + lane < a.n ? p.sub[c0 + 32 * h + lane] : 0.f;
        __syncwarp();
      }
      for (int64_t g = g0; g < g1; ++g) {
        const int s = qs;
        const uint32_t sph = qph;
        const bool mine = turn == warp;
        if (++qs == S) {
          qs = 0;
          qph ^= 1u;
        }
        if (++turn == kConsumers) turn = 0;
        if (!mine) continue;
        // Stage s's rounds alternate between this warp and at most one other
        // (2 x the stage count is a multiple of the consumer warps), so the
        // round before this one may be the other warp's and its load may still
        // be in flight, when a parity wait on full[s] would pass a phase early.
        // Its consumption on empty[s] comes first: at once for the first round
        // and for a round this warp consumed itself.
        if (!mbar_wait(&empty[s], sph ^ 1u, abort_flag)) break;
        if (!mbar_wait(&full[s], sph, abort_flag)) break;
        const uint8_t* tile = ring + s * a.stage_bytes;
#pragma unroll 1
        for (int sub_step = 0; sub_step < 4; ++sub_step) {
          const int r = 16 * sub_step + i;
          const int64_t R = g * kTileRows + r;
          float v[32];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int phys = (4 * u + k) ^ (r & 7);
            unpack8(*reinterpret_cast<const uint4*>(tile + r * 128 + phys * 16), v + 8 * k);
          }
          const bool ok = R < a.m && unit_ok;
          float ds = 0.f;
          if (ok) {
            if (SUB) {
#pragma unroll
              for (int j = 0; j < 32; j += 4) {
                const float4 m = *reinterpret_cast<const float4*>(&wsub[warp][u][j]);
                v[j] = __fsub_rn(v[j], m.x);
                v[j + 1] = __fsub_rn(v[j + 1], m.y);
                v[j + 2] = __fsub_rn(v[j + 2], m.z);
                v[j + 3] = __fsub_rn(v[j + 3], m.w);
              }
            }
            if (p.r_tap) {
              float* tp = p.r_tap + R * p.tap_ld + cu;
#pragma unroll
              for (int j = 0; j < 32; j += 4) *reinterpret_cast<float4*>(tp + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
            }
            const int64_t un = cu / 32;           // the unit's index along the row
            uint4* dst = reinterpret_cast<uint4*>(p.codes + R * outer_ld + un * 16);
            if (FMT == METIS_NVFP4) {
              uint64_t pk0, pk1;
              float d0, d1;
              const uint32_t k0 = quant_block_nv_tab<SUM>(v, s_t, enc_tab, pk0, d0);
              const uint32_t k1 = quant_block_nv_tab<SUM>(v + 16, s_t, enc_tab, pk1, d1);
              if (SUM) ds = d0 + d1;
              *dst = make_uint4(static_cast<uint32_t>(pk0), static_cast<uint32_t>(pk0 >> 32), static_cast<uint32_t>(pk1),
                                static_cast<uint32_t>(pk1 >> 32));
              *reinterpret_cast<uint16_t*>(p.scales + tc_scale_offset(R, 2 * un, p.scale_cols)) =
                  static_cast<uint16_t>(k0 | (k1 << 8));
              if (p.scales_linear) {
                p.scales_linear[R * (p.inner / 16) + 2 * un] = static_cast<uint8_t>(k0);
                p.scales_linear[R * (p.inner / 16) + 2 * un + 1] = static_cast<uint8_t>(k1);
              }
            } else {
              uint64_t pk[2];
              const uint32_t k0 = quant_block_mx<SUM>(v, pk, ds);
              *dst = make_uint4(static_cast<uint32_t>(pk[0]), static_cast<uint32_t>(pk[0] >> 32),
                                static_cast<uint32_t>(pk[1]), static_cast<uint32_t>(pk[1] >> 32));
              p.scales[tc_scale_offset(R, un, p.scale_cols)] = static_cast<uint8_t>(k0);
              if (p.scales_linear) p.scales_linear[R * (p.inner / 32) + un] = static_cast<uint8_t>(k0);
            }
          }  // ok
          if (SUM) {
            // the strip's two units of row R: lanes 2i and 2i + 1 (0 for a unit past n)
            const float other = __shfl_xor_sync(0xFFFFFFFFu, ds, 1);
            if (u == 0 && R < a.m) p.partial_sums[R * p.ngroups + strip] = ds + other;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);   // every value read from the stage has been used
      }
    } else {
      // ---- blocks along rows
      constexpr int kBlk = FMT == METIS_NVFP4 ? 16 : 32;
      constexpr int kLanesPerCol = kTileRows / kBlk;        // 4 or 2 blocks per tile column
      constexpr int kGroups = 32 / kLanesPerCol;            // 8 or 16 column groups of 8
      const int b = lane / kGroups, cg = lane % kGroups;
      const int row_bytes = a.strip_cols * 2;
      // lane-indexed shared copies (conflict-free), so that the column loop
      // below needs no register arrays indexed by a runtime column
      float (*subc)[32] = wcol[warp][0];
      float (*colsum)[32] = wcol[warp][1];
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        colsum[j][lane] = 0.f;
        const int64_t C = c0 + 8 * cg + j;
        subc[j][lane] = (SUB && C < a.n) ? p.sub[C] : 0.f;
      }
      __syncwarp();
      for (int64_t g = g0; g < g1; ++g) {
        const int s = qs;
        const uint32_t sph = qph;
        const bool mine = turn == warp;
        if (++qs == S) {
          qs = 0;
          qph ^= 1u;
        }
        if (++turn == kConsumers) turn = 0;
        if (!mine) continue;
        // Stage s's rounds alternate between this warp and at most one other
        // (2 x the stage count is a multiple of the consumer warps), so the
        // round before this one may be the other warp's and its load may still
        // be in flight, when a parity wait on full[s] would pass a phase early.
        // Its consumption on empty[s] comes first: at once for the first round
        // and for a round this warp consumed itself.
        if (!mbar_wait(&empty[s], sph ^ 1u, abort_flag)) break;
        if (!mbar_wait(&full[s], sph, abort_flag)) break;
        const uint8_t* tile = ring + s * a.stage_bytes;
        const int64_t rb = g * kTileRows + kBlk * b;        // the block's first X row
        const bool rows_ok = rb + kBlk <= a.m;               // m is a multiple of the block
        // NVFP4: two passes over 4 columns (an 8-byte word per row, 16 rows);
        // MXFP4: four passes over 2 columns (a 4-byte word per row, 32
        // rows).  The block's rows stay packed (2 bf16 per register).
        constexpr int kCols = kBlk == 16 ? 4 : 2;
        constexpr int kWords = kCols / 2;
#pragma unroll 1
        for (int h = 0; h < 8 / kCols; ++h) {
          uint32_t raw[kBlk][kWords];
#pragma unroll
          for (int i = 0; i < kBlk; ++i) {
            const uint8_t* src = tile + (kBlk * b + i) * row_bytes + cg * 16 + h * 2 * kCols;
            if (kCols == 4) {
              const uint2 w = *reinterpret_cast<const uint2*>(src);
              raw[i][0] = w.x;
              raw[i][kWords - 1] = w.y;
            } else {
              raw[i][0] = *reinterpret_cast<const uint32_t*>(src);
            }
          }
#pragma unroll
          for (int j = 0; j < kCols; ++j) {
            const int jc = h * kCols + j;                    // column within the lane's 8
            const int64_t C = c0 + 8 * cg + jc;
            float v[kBlk];
#pragma unroll
            for (int i = 0; i < kBlk; ++i) {
              const uint32_t w = raw[i][j >> 1];
              const float x = __uint_as_float((j & 1) ? (w & 0xFFFF0000u) : (w << 16));
              v[i] = SUB ? __fsub_rn(x, subc[jc][lane]) : x;
            }
            float ds = 0.f;
            if (C < a.n && rows_ok) {
              if (p.r_tap) {
#pragma unroll
                for (int i = 0; i < kBlk; ++i) p.r_tap[(rb + i) * p.tap_ld + C] = v[i];
              }
              uint8_t* dst = p.codes + C * outer_ld + rb / 2;
              const int64_t sc = rb / kBlk;
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
              p.scales[tc_scale_offset(C, sc, p.scale_cols)] = static_cast<uint8_t>(code);
              if (p.scales_linear) p.scales_linear[C * (p.inner / kBlk) + sc] = static_cast<uint8_t>(code);
            }
            if (SUM) {
              // the column's blocks of this tile: lanes cg, cg + kGroups, ...
#pragma unroll
              for (int off = kGroups; off < 32; off <<= 1) ds += __shfl_xor_sync(0xFFFFFFFFu, ds, off);
              colsum[jc][lane] += ds;
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);   // every value read from the stage has been used
      }
      if (SUM && b == 0) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int64_t C = c0 + 8 * cg + j;
          if (C < a.n) p.partial_sums[C * p.ngroups + run * kConsumers + warp] = colsum[j][lane];
        }
      }
    }
  }
  if (threadIdx.x == 0 && *abort_flag) report(a.dev_status, METIS_DEV_TIMEOUT);
}

template <int FMT, bool SUM, bool SUB, int AXIS>
void launch_t(const TmaQuantArgs& a, const CUtensorMap& map, int grid, size_t smem, cudaStream_t s) {
  const void* fn = reinterpret_cast<const void*>(quantize_tma_kernel<FMT, SUM, SUB, AXIS>);
  if (!ensure_smem(fn, smem)) return;
  quantize_tma_kernel<FMT, SUM, SUB, AXIS><<<grid, kQThreads, smem, s>>>(a, map);
}

template <int FMT, int AXIS>
void launch_f(const TmaQuantArgs& a, const CUtensorMap& map, int grid, size_t smem, cudaStream_t s) {
  const bool sum = a.p.partial_sums != nullptr, sub = a.p.sub != nullptr;
  if (sum && sub) launch_t<FMT, true, true, AXIS>(a, map, grid, smem, s);
  else if (sum) launch_t<FMT, true, false, AXIS>(a, map, grid, smem, s);
  else if (sub) launch_t<FMT, false, true, AXIS>(a, map, grid, smem, s);
  else launch_t<FMT, false, false, AXIS>(a, map, grid, smem, s);
}

}  // namespace

int64_t quantize_tma_groups(const QuantParams& p, int axis, int sms);

bool quantize_tma_ok(const QuantParams& p, int axis, int sms) {
  if (p.dtype != METIS_BF16) return false;
  if ((reinterpret_cast<uintptr_t>(p.X) & 15u) || (p.ld * 2) % 16) return false;
  // X's columns: inner for axis 1, outer for axis 0 (16-byte TMA rows)
  const int64_t n = axis == 1 ? p.inner : p.outer;
  if (n % 8 != 0 || (axis == 1 && p.inner % 32 != 0)) return false;
  // blocks along columns without a subtraction or sums: the register-prefetch
  // kernel (quantize.cu), with more warps resident, is faster
  if (axis == 1 && !p.sub && !p.partial_sums) return false;
  // the partial sums fit the workspace (outer x ceil(inner / 64) floats)
  return !p.partial_sums || quantize_tma_groups(p, axis, sms) <= (p.inner + 63) / 64;
}

int64_t quantize_tma_groups(const QuantParams& p, int axis, int sms) {
  // partial sums per outer index: axis 1 one per 64-column strip; axis 0 one
  // per (run, consumer warp)
  if (axis == 1) return (p.inner + 63) / 64;
  const int64_t m = p.inner, n = p.outer;
  const int cols = p.fmt == METIS_MXFP4 ? 128 : 64;
  const int64_t strips = (n + cols - 1) / cols, ntiles = (m + kTileRows - 1) / kTileRows;
  int64_t runs = imax64(1, imin64(ntiles, (4 * static_cast<int64_t>(sms) + strips - 1) / strips));
  const int64_t run_tiles = (ntiles + runs - 1) / runs;
  runs = (ntiles + run_tiles - 1) / run_tiles;
  return runs * kConsumers;
}

void launch_quantize_tma(QuantParams p, int axis, int sms, int32_t* dev_status, cudaStream_t s) {
  TmaQuantArgs a{};
  const bool mx = p.fmt == METIS_MXFP4;
  a.m = axis == 1 ? p.outer : p.inner;
  a.n = axis == 1 ? p.inner : p.outer;
  a.strip_cols = (axis == 0 && mx) ? 128 : 64;
  a.stage_bytes = kTileRows * a.strip_cols * 2;
  a.stages = ring_bytes(axis) / a.stage_bytes;
  // the consumers' waits assume a stage's rounds alternate between at most two warps
  if ((2 * a.stages) % kConsumers != 0) {
    fail(METIS_ERR_ARG, "quantize ring stages");
    return;
  }
  a.strips = (a.n + a.strip_cols - 1) / a.strip_cols;
  a.ntiles = (a.m + kTileRows - 1) / kTileRows;
  // about four items per CTA slot (two CTAs per SM) for balance
  int64_t runs = imax64(1, imin64(a.ntiles, (4 * static_cast<int64_t>(sms) + a.strips - 1) / a.strips));
  a.run_tiles = (a.ntiles + runs - 1) / runs;
  a.runs = (a.ntiles + a.run_tiles - 1) / a.run_tiles;
  if (p.partial_sums) p.ngroups = quantize_tma_groups(p, axis, sms);
  a.p = p;
  a.dev_status = dev_status;
  CUtensorMap map;
  const uint64_t dims[2] = {static_cast<uint64_t>(a.n), static_cast<uint64_t>(a.m)};
  const uint64_t strides[1] = {static_cast<uint64_t>(p.ld) * 2};
  const uint32_t box[2] = {static_cast<uint32_t>(a.strip_cols), static_cast<uint32_t>(kTileRows)};
  if (encode_tensor_map(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.X, dims, strides, box,
                        axis == 1 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS) {
    fail(METIS_ERR_CUDA, "quantize tensor map");
    return;
  }
  const int grid = static_cast<int>(imin64(a.strips * a.runs, ctas_per_sm(axis) * static_cast<int64_t>(sms)));
  const size_t smem = static_cast<size_t>(a.stages) * a.stage_bytes + 1024;
  if (axis == 1) {
    if (mx) launch_f<METIS_MXFP4, 1>(a, map, grid, smem, s);
    else launch_f<METIS_NVFP4, 1>(a, map, grid, smem, s);
  } else {
    if (mx) launch_f<METIS_MXFP4, 0>(a, map, grid, smem, s);
    else launch_f<METIS_NVFP4, 0>(a, map, grid, smem, s);
  }
}

}  // namespace metis
