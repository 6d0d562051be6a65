// Fused residual + FP4 quantization: R = A - U diag(S) V^T, tile by tile,
// quantized along either or both block axes in the same pass.
//
// Source: SII release on Metis, section 2.4 item 1 (the long-tail residual is
// quantized on its own after the dominant part is split off) and section 2.3
// / Fig. 3 (block-wise scales set by the block maximum); formats from the
// feature list (MXFP4 / NVFP4).
//
// Persistent, warp-specialized kernel; one CTA per SM walks a contiguous run
// of 128 x BN tiles of A in row-band order (BN = 128 where two stages of that
// width fit in shared memory, else 64; a wider tile halves the MMA
// instructions per output, and the MMA warp's issue rate is what bounds the
// pass):
//   warp 0      TMA producer: the band's rows of U (hi, lo; reloaded only
//               when the band changes) and, per tile, the BN rows of
//               W = V diag(S) (hi, lo) and the 128 x BN tile of A, into a ring
//               of shared-memory stages;
//   warp 1      TMEM owner and MMA issuer: U_hi W_hi + U_hi W_lo + U_lo W_hi as
//               kind::f16 MMAs (M 128, N BN) into one of four TMEM
//               accumulators, so L = U S V^T to ~2^-16 relative;
//   warps 2-9   epilogue, 32 rows x 32 columns per chunk (BN / 64 chunks
//               each): L from TMEM, A from the
//               swizzled stage, R = fl32(a - l); then either the tensor
//               maximum of |R| (the NVFP4 pre-pass) or the FP4 codes: blocks
//               along n straight from registers, blocks along m through a
//               per-warp 32 x 32 shared-memory transpose, plus an optional
//               float32 tap of R.
// Loads of the next tiles and MMAs overlap the epilogue of the current one.
// HBM-bound: A is read once per pass (twice for NVFP4) and FP4 codes plus
// scales are written once per quantized axis.
#include "abi_common.h"
#include "common.cuh"
#include "fp4_block.cuh"
#include "residual_quant.h"

namespace metis {

namespace {

MDEV bool wait_ns(uint64_t* bar, uint32_t parity, uint64_t ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > ns) return false;
  }
  return true;
}

// Quantize n (32 or 64) values along the block axis: outer index o, first
// element at inner offset i0 (a multiple of 32).
MDEV void emit(const float* v, int n, int fmt, float s_t, const float* enc_tab, uint8_t* codes, uint8_t* scales,
               int64_t scale_cols, int64_t inner, int64_t o, int64_t i0) {
  uint8_t* dst = codes + o * (inner / 2) + i0 / 2;
  if (fmt == METIS_NVFP4) {
    uint64_t pk[4] = {0, 0, 0, 0};
    uint32_t sc = 0;
    const int nb = n / 16;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      if (b < nb) {
        sc |= quant_block_nv_tab(v + 16 * b, s_t, enc_tab, pk[b]) << (8 * b);
      }
    }
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(static_cast<uint32_t>(pk[0]), static_cast<uint32_t>(pk[0] >> 32),
                                                  static_cast<uint32_t>(pk[1]), static_cast<uint32_t>(pk[1] >> 32));
    if (nb > 2)
      reinterpret_cast<uint4*>(dst)[1] = make_uint4(static_cast<uint32_t>(pk[2]), static_cast<uint32_t>(pk[2] >> 32),
                                                    static_cast<uint32_t>(pk[3]), static_cast<uint32_t>(pk[3] >> 32));
    const int64_t c0 = i0 / 16;
    if (nb > 2)
      *reinterpret_cast<uint32_t*>(scales + tc_scale_offset(o, c0, scale_cols)) = sc;
    else
      *reinterpret_cast<uint16_t*>(scales + tc_scale_offset(o, c0, scale_cols)) = static_cast<uint16_t>(sc);
  } else {
    uint64_t pk[4] = {0, 0, 0, 0};
    uint32_t sc = 0;
    const int nb = n / 32;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      if (b < nb) {
        float ds;
        sc |= quant_block_mx(v + 32 * b, pk + 2 * b, ds) << (8 * b);
      }
    }
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(static_cast<uint32_t>(pk[0]), static_cast<uint32_t>(pk[0] >> 32),
                                                  static_cast<uint32_t>(pk[1]), static_cast<uint32_t>(pk[1] >> 32));
    if (nb > 1)
      reinterpret_cast<uint4*>(dst)[1] = make_uint4(static_cast<uint32_t>(pk[2]), static_cast<uint32_t>(pk[2] >> 32),
                                                    static_cast<uint32_t>(pk[3]), static_cast<uint32_t>(pk[3] >> 32));
    const int64_t c0 = i0 / 32;
    if (nb > 1)
      *reinterpret_cast<uint16_t*>(scales + tc_scale_offset(o, c0, scale_cols)) = static_cast<uint16_t>(sc);
    else
      scales[tc_scale_offset(o, c0, scale_cols)] = static_cast<uint8_t>(sc);
  }
}


constexpr int kBM = 128;         // tile rows (one band)
constexpr int kAccBufs = 4;      // TMEM accumulators of BN columns
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr int kMaxStages = 6;
constexpr int kSmemLimit = 232448;  // opt-in shared memory per CTA on sm_100
constexpr int kTransposeBytes = kEpiWarps * 32 * 33 * 4;

struct Layout {
  int bn;           // tile columns: 128, or 64 where two such stages do not fit
  int chunks;       // kp / 64
  int u_bytes;      // U hi + lo
  int w_bytes;      // per stage: W hi + lo
  int a_bytes;      // per stage: the A tile
  int stages;
  int total;        // dynamic shared memory including 1024 B of alignment slack
};

// `transpose`: the column-axis codes need the per-warp transpose buffer;
// without them its space goes to more stages.
__host__ __device__ inline Layout layout_bn(int kp, int dtype, bool transpose, int bn) {
  Layout l{};
  l.bn = bn;
  l.chunks = kp / 64;
  l.u_bytes = 2 * l.chunks * kBM * 128;
  l.w_bytes = 2 * l.chunks * bn * 128;
  l.a_bytes = kBM * bn * (dtype == METIS_BF16 ? 2 : 4);
  const int fixed = 1024 + l.u_bytes + (transpose ? kTransposeBytes : 0) + 1024;  // barriers 256 B, encode table 512 B
  int st = (kSmemLimit - fixed) / (l.w_bytes + l.a_bytes);
  l.stages = st > kMaxStages ? kMaxStages : st;
  l.total = fixed + l.stages * (l.w_bytes + l.a_bytes);
  return l;
}

__host__ __device__ inline Layout layout(int kp, int dtype, bool transpose) {
  const Layout wide = layout_bn(kp, dtype, transpose, 128);
  return wide.stages >= 2 ? wide : layout_bn(kp, dtype, transpose, 64);
}

__global__ void __launch_bounds__(kThreads, 1) residual_quant_kernel(const ResidualParams p,
                                                                     const __grid_constant__ CUtensorMap tmUhi,
                                                                     const __grid_constant__ CUtensorMap tmUlo,
                                                                     const __grid_constant__ CUtensorMap tmWhi,
                                                                     const __grid_constant__ CUtensorMap tmWlo,
                                                                     const __grid_constant__ CUtensorMap tmA) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const bool transpose = p.c_codes != nullptr;
  const Layout lo = layout(p.kp, p.dtype, transpose);
  const int S = lo.stages;
  uint8_t* sUhi = smem;
  uint8_t* sUlo = sUhi + lo.u_bytes / 2;
  uint8_t* sStage = smem + lo.u_bytes;
  const int stage_bytes = lo.w_bytes + lo.a_bytes;
  float* tstage = reinterpret_cast<float*>(sStage + S * stage_bytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(tstage) + (transpose ? kTransposeBytes : 0));
  uint64_t* full = bars;                           // [kMaxStages]
  uint64_t* empty = full + kMaxStages;             // [kMaxStages]
  uint64_t* acc_full = empty + kMaxStages;         // [kAccBufs]
  uint64_t* acc_empty = acc_full + kAccBufs;       // [kAccBufs]
  uint64_t* u_full = acc_empty + kAccBufs;
  uint64_t* u_empty = u_full + 1;
  uint64_t* drain = u_empty + 1;
  uint32_t* tmem_sh = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_sh + 1);
  float* enc_tab = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 256);  // NVFP4 encode factors

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kEpiWarps);
    }
    for (int i = 0; i < kAccBufs; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kEpiWarps);
    }
    mbar_init(u_full, 1);
    mbar_init(u_empty, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmUhi);
    prefetch_tensormap(&tmUlo);
    prefetch_tensormap(&tmWhi);
    prefetch_tensormap(&tmWlo);
    prefetch_tensormap(&tmA);
  }
  if (warp == 1) {
    tmem_alloc(tmem_sh, static_cast<uint32_t>(kAccBufs * lo.bn));
    tmem_relinquish();
  }
  if (p.mode == 1 && p.fmt == METIS_NVFP4) nv_enc_table(nv_tensor_scale(__uint_as_float(*p.amax_bits)), enc_tab);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_sh;

  // this CTA's contiguous run of tiles, in row-band order
  const int bn = lo.bn;
  const int nt = static_cast<int>((p.n + bn - 1) / bn);
  const int total = static_cast<int>((p.m + kBM - 1) / kBM) * nt;
  const int per = (total + gridDim.x - 1) / gridDim.x;
  const int t0 = blockIdx.x * per;
  const int t1 = min(total, t0 + per);
  const bool f32 = p.dtype == METIS_F32;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0, issued = 0, u_loads = 0, cur_tm = -1;
      uint32_t ph = 0, uph = 0;
      for (int t = t0; t < t1; ++t) {
        const int tm = t / nt, tn = t - tm * nt;
        if (tm != cur_tm) {
          if (cur_tm >= 0) {
            if (!mbar_wait(u_empty, uph, abort_flag)) break;
            uph ^= 1u;
          }
          mbar_arrive_expect_tx(u_full, lo.u_bytes);
          for (int c = 0; c < lo.chunks; ++c) {
            tma_load_2d(sUhi + c * kBM * 128, &tmUhi, u_full, 64 * c, tm * kBM);
            tma_load_2d(sUlo + c * kBM * 128, &tmUlo, u_full, 64 * c, tm * kBM);
          }
          ++u_loads;
          cur_tm = tm;
        }
        if (!mbar_wait(&empty[stage], ph ^ 1u, abort_flag)) break;
        uint8_t* sW = sStage + stage * stage_bytes;
        uint8_t* sA = sW + lo.w_bytes;
        mbar_arrive_expect_tx(&full[stage], stage_bytes);
        for (int c = 0; c < lo.chunks; ++c) {
          tma_load_2d(sW + c * bn * 128, &tmWhi, &full[stage], 64 * c, tn * bn);
          tma_load_2d(sW + (lo.chunks + c) * bn * 128, &tmWlo, &full[stage], 64 * c, tn * bn);
        }
        // A: boxes of 128 bytes per row (32 float32 or 64 bf16 columns)
        const int box_cols = f32 ? 32 : 64;
        for (int b = 0; b < bn / box_cols; ++b)
          tma_load_2d(sA + b * kBM * 128, &tmA, &full[stage], tn * bn + box_cols * b, tm * kBM);
        ++issued;
        if (++stage == S) {
          stage = 0;
          ph ^= 1u;
        }
      }
      if (*abort_flag) {
        // let copies already in flight land before the CTA exits
        int st = stage;
        uint32_t pp = ph;
        for (int i = 0; i < min(issued, S); ++i) {
          if (--st < 0) {
            st = S - 1;
            pp ^= 1u;
          }
          wait_ns(&full[st], pp, 100000000ull);
        }
        if (u_loads > 0) wait_ns(u_full, static_cast<uint32_t>(u_loads - 1) & 1u, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0, acc = 0, bands = 0, cur_tm = -1;
      uint32_t ph = 0, aph = 0;
      const uint32_t idesc = idesc_bf16(kBM, bn, false, false);
      for (int t = t0; t < t1; ++t) {
        const int tm = t / nt;
        if (tm != cur_tm) {
          if (cur_tm >= 0) tc_commit(u_empty);  // the old U is free once these MMAs retire
          if (!mbar_wait(u_full, static_cast<uint32_t>(bands) & 1u, abort_flag)) break;
          ++bands;
          cur_tm = tm;
        }
        if (!mbar_wait(&acc_empty[acc], aph ^ 1u, abort_flag)) break;
        if (!mbar_wait(&full[stage], ph, abort_flag)) break;
        tc_fence_after();
        uint8_t* sW = sStage + stage * stage_bytes;
        const uint32_t d = tmem + static_cast<uint32_t>(acc * bn);
        uint32_t accumulate = 0;
        for (int c = 0; c < lo.chunks; ++c) {
          const uint64_t uh = make_sdesc(smem_u32(sUhi + c * kBM * 128), 16, 1024, kSwizzle128B);
          const uint64_t ul = make_sdesc(smem_u32(sUlo + c * kBM * 128), 16, 1024, kSwizzle128B);
          const uint64_t wh = make_sdesc(smem_u32(sW + c * bn * 128), 16, 1024, kSwizzle128B);
          const uint64_t wl = make_sdesc(smem_u32(sW + (lo.chunks + c) * bn * 128), 16, 1024, kSwizzle128B);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t o = static_cast<uint64_t>(2 * j);  // 32 bytes of K per step
            mma_bf16(d, uh + o, wh + o, idesc, accumulate);
            accumulate = 1;
            mma_bf16(d, uh + o, wl + o, idesc, 1);
            mma_bf16(d, ul + o, wh + o, idesc, 1);
          }
        }
        tc_commit(&acc_full[acc]);
        if (++stage == S) {
          stage = 0;
          ph ^= 1u;
        }
        if (++acc == kAccBufs) {
          acc = 0;
          aph ^= 1u;
        }
      }
      if (*abort_flag) {
        // wait for MMAs already issued before the TMEM is freed
        tc_commit(drain);
        wait_ns(drain, 0, 100000000ull);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;             // TMEM lane quadrant: rows 32 q .. 32 q + 31
    const int h = (warp - 2) >> 2;      // chunk parity: columns 32 h .. (and 32 (h + 2) .. for BN = 128)
    float* my_t = tstage + (warp - 2) * 32 * 33;
    float s_t = 1.f;
    if (p.mode == 1 && p.fmt == METIS_NVFP4) s_t = nv_tensor_scale(__uint_as_float(*p.amax_bits));
    if (p.mode == 1 && p.fmt == METIS_NVFP4 && blockIdx.x == 0 && warp == 2 && lane == 0) {
      if (p.ts_rows) *p.ts_rows = s_t;
      if (p.ts_cols) *p.ts_cols = s_t;
    }
    float amax = 0.f;
    int stage = 0, acc = 0;
    uint32_t ph = 0, aph = 0;
    const int nc = bn / 64;             // 32-column chunks of this warp: h, h + 2 (BN = 128)
    for (int t = t0; t < t1; ++t) {
      const int tm = t / nt, tn = t - tm * nt;
      if (!mbar_wait(&acc_full[acc], aph, abort_flag)) break;
      tc_fence_after();
      uint32_t L[2][32];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        if (cc < nc) {
          const uint32_t col = static_cast<uint32_t>(acc * bn + 32 * (h + 2 * cc));
          tmem_ld16(tmem + (static_cast<uint32_t>(32 * q) << 16) + col, L[cc]);
          tmem_ld16(tmem + (static_cast<uint32_t>(32 * q) << 16) + col + 16, L[cc] + 16);
        }
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (!mbar_wait(&full[stage], ph, abort_flag)) break;  // the A tile has landed
      const int r = 32 * q + lane;                          // row within the tile
      const uint8_t* sA = sStage + stage * stage_bytes + lo.w_bytes;
      float v[2][32];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        if (cc >= nc) continue;
        const int ch = h + 2 * cc;                          // columns 32 ch .. 32 ch + 31
        if (f32) {
          const uint8_t* base = sA + ch * kBM * 128 + r * 128;  // box ch holds columns 32 ch ..
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 f = *reinterpret_cast<const float4*>(base + ((j ^ (r & 7)) << 4));
            v[cc][4 * j] = f.x;
            v[cc][4 * j + 1] = f.y;
            v[cc][4 * j + 2] = f.z;
            v[cc][4 * j + 3] = f.w;
          }
        } else {
          const uint8_t* base = sA + (ch >> 1) * kBM * 128 + r * 128;  // box ch / 2 holds columns 64 (ch / 2) ..
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const int j = 4 * (ch & 1) + jj;
            const uint4 u = *reinterpret_cast<const uint4*>(base + ((j ^ (r & 7)) << 4));
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              v[cc][8 * jj + 2 * i] = __uint_as_float(w[i] << 16);
              v[cc][8 * jj + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
            }
          }
        }
        // the residual: using every loaded value before the stage is handed
        // back means the shared-memory reads have returned (a load whose
        // value is first used after the arrive could still be reading while
        // the next TMA copy lands in the stage)
#pragma unroll
        for (int j = 0; j < 32; ++j) v[cc][j] = __fsub_rn(v[cc][j], __uint_as_float(L[cc][j]));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      if (++stage == S) {
        stage = 0;
        ph ^= 1u;
      }
      if (++acc == kAccBufs) {
        acc = 0;
        aph ^= 1u;
      }
      const int64_t row0 = static_cast<int64_t>(tm) * kBM + 32 * q;
      const int64_t row = row0 + lane;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        if (cc >= nc) continue;
        const int64_t col0 = static_cast<int64_t>(tn) * bn + 32 * (h + 2 * cc);
        if (row0 >= p.m || col0 >= p.n) continue;  // m, n are multiples of 32: whole warp
        const float* vc = v[cc];
        if (p.mode == 0) {
#pragma unroll
          for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(vc[j]));
          continue;
        }
        if (p.r_tap) {
          float* tp = p.r_tap + row * p.n + col0;
#pragma unroll
          for (int j = 0; j < 32; j += 4) *reinterpret_cast<float4*>(tp + j) = make_float4(vc[j], vc[j + 1], vc[j + 2], vc[j + 3]);
        }
        if (p.r_codes) emit(vc, 32, p.fmt, s_t, enc_tab, p.r_codes, p.r_scales, p.r_scale_cols, p.n, row, col0);
        if (p.c_codes) {
          // the warp's 32 rows x 32 columns, transposed through shared memory
#pragma unroll
          for (int j = 0; j < 32; ++j) my_t[lane * 33 + j] = vc[j];
          __syncwarp();
          float col[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) col[i] = my_t[i * 33 + lane];
          __syncwarp();
          emit(col, 32, p.fmt, s_t, enc_tab, p.c_codes, p.c_scales, p.c_scale_cols, p.m, col0 + lane, row0);
        }
      }
    }
    if (p.mode == 0) {
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      if (lane == 0) atomicMax(p.amax_bits, __float_as_uint(amax));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(kAccBufs * lo.bn));
  }
  if (threadIdx.x == 0 && *abort_flag) report(p.dev_status, METIS_DEV_TIMEOUT);
}

// The split's factors after the sign choice, in one pass over U (m x k) and
// V (n x k): both are multiplied by sign (in place); U and V diag(S) are
// written as bf16 hi / lo pairs [rows][kp] (zero padded, when hi pointers are
// given), and the tensor maxima of |U| and |V| are atomically maxed into
// amax[0], amax[1] (when given; the NVFP4 quantizer of U and V reads them).
__global__ void __launch_bounds__(256) factor_finish_kernel(float* U, int64_t m, float* V, int64_t n, int k,
                                                            const float* sign, const float* S, int kp,
                                                            __nv_bfloat16* u_hi, __nv_bfloat16* u_lo,
                                                            __nv_bfloat16* w_hi, __nv_bfloat16* w_lo,
                                                            unsigned* amax) {
  // thread (c, ry): column c of rows ry, ry + blockDim.y, ... of this CTA's
  // share (U's rows first, then V's); one atomic per CTA and matrix
  __shared__ float red[2][32];
  const int c = threadIdx.x;
  const int nthr = blockDim.x * blockDim.y, tid = threadIdx.y * blockDim.x + threadIdx.x;
  float mu = 0.f, mv = 0.f;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * blockDim.y + threadIdx.y; row < m + n;
       row += static_cast<int64_t>(gridDim.x) * blockDim.y) {
    const bool isu = row < m;
    const int64_t r = isu ? row : row - m;
    float w = 0.f;
    if (c < k) {
      float* x = (isu ? U : V) + r * k + c;
      const float v = *x * sign[c];
      *x = v;
      if (isu) {
        mu = fmaxf(mu, fabsf(v));
        w = v;
      } else {
        mv = fmaxf(mv, fabsf(v));
        w = __fmul_rn(v, S[c]);
      }
    }
    __nv_bfloat16* hi = isu ? u_hi : w_hi;
    __nv_bfloat16* lo = isu ? u_lo : w_lo;
    if (hi && c < kp) {
      const __nv_bfloat16 h = __float2bfloat16_rn(w);
      hi[r * kp + c] = h;
      lo[r * kp + c] = __float2bfloat16_rn(__fsub_rn(w, __bfloat162float(h)));
    }
  }
  if (amax) {
    for (int o = 16; o > 0; o >>= 1) {
      mu = fmaxf(mu, __shfl_xor_sync(0xFFFFFFFFu, mu, o));
      mv = fmaxf(mv, __shfl_xor_sync(0xFFFFFFFFu, mv, o));
    }
    if ((tid & 31) == 0) {
      red[0][tid >> 5] = mu;
      red[1][tid >> 5] = mv;
    }
    __syncthreads();
    if (tid == 0) {
      for (int w = 1; w < nthr / 32; ++w) {
        mu = fmaxf(mu, red[0][w]);
        mv = fmaxf(mv, red[1][w]);
      }
      if (mu > 0.f) atomicMax(amax, __float_as_uint(mu));
      if (mv > 0.f) atomicMax(amax + 1, __float_as_uint(mv));
    }
  }
}

CUresult map_kmajor(CUtensorMap* m, const void* base, int64_t rows, int kp, uint32_t box_rows) {
  const uint64_t dims[2] = {static_cast<uint64_t>(kp), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(kp) * 2};
  const uint32_t box[2] = {64, box_rows};
  return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B);
}

// A (m x n, row stride lda): boxes of 128 bytes of a row x 128 rows.
CUresult map_a(CUtensorMap* m, const ResidualParams& p) {
  const bool bf = p.dtype == METIS_BF16;
  const uint64_t dims[2] = {static_cast<uint64_t>(p.n), static_cast<uint64_t>(p.m)};
  const uint64_t strides[1] = {static_cast<uint64_t>(p.lda) * (bf ? 2 : 4)};
  const uint32_t box[2] = {bf ? 64u : 32u, static_cast<uint32_t>(kBM)};
  return encode_tensor_map(m, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, p.A, dims,
                           strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

void launch_factor_finish(float* U, int64_t m, float* V, int64_t n, int k, const float* sign, const float* S, int kp,
                          __nv_bfloat16* u_hi, __nv_bfloat16* u_lo, __nv_bfloat16* w_hi, __nv_bfloat16* w_lo,
                          unsigned* amax, int sms, cudaStream_t s) {
  const int cols = ((kp > k ? kp : k) + 31) / 32 * 32;  // <= 128
  const dim3 block(cols, 256 / cols);
  int64_t grid = (m + n + block.y - 1) / block.y;
  if (grid > 2 * sms) grid = 2 * sms;  // a few atomics per matrix, not one per warp
  factor_finish_kernel<<<static_cast<unsigned>(grid), block, 0, s>>>(U, m, V, n, k, sign, S, kp, u_hi, u_lo, w_hi,
                                                                     w_lo, amax);
}

metis_status run_residual_quant(const ResidualParams& p, const ResidualOperands& o, cudaStream_t s) {
  const Layout lo = layout(p.kp, p.dtype, p.c_codes != nullptr);
  CUtensorMap uh, ul, wh, wl, ta;
  if (map_kmajor(&uh, o.u_hi, p.m, p.kp, kBM) != CUDA_SUCCESS || map_kmajor(&ul, o.u_lo, p.m, p.kp, kBM) != CUDA_SUCCESS ||
      map_kmajor(&wh, o.w_hi, p.n, p.kp, lo.bn) != CUDA_SUCCESS || map_kmajor(&wl, o.w_lo, p.n, p.kp, lo.bn) != CUDA_SUCCESS ||
      map_a(&ta, p) != CUDA_SUCCESS)
    return fail(METIS_ERR_CUDA, "residual tensor map");
  if (lo.stages < 2) return fail(METIS_ERR_SHAPE, "residual", "factor rank too large for the shared-memory stages");
  if (!ensure_smem(reinterpret_cast<const void*>(residual_quant_kernel), lo.total))
    return fail(METIS_ERR_CUDA, "residual shared-memory attribute");
  const int64_t tiles = ((p.m + kBM - 1) / kBM) * ((p.n + lo.bn - 1) / lo.bn);
  const int sms = device_sm_count();
  const int64_t per = (tiles + sms - 1) / sms;
  const unsigned grid = static_cast<unsigned>((tiles + per - 1) / per);
  residual_quant_kernel<<<grid, kThreads, lo.total, s>>>(p, uh, ul, wh, wl, ta);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(METIS_ERR_CUDA, "residual_quant launch", cudaGetErrorString(e));
  return METIS_OK;
}

}  // namespace metis
