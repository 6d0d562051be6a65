// Fused residual + FP4 quantization: R = A - U diag(S) V^T, tile by tile,
// quantized along both block axes in the same pass.
//
// Source: SII release on Metis, section 2.4 item 1 (the long-tail residual is
// quantized on its own after the dominant part is split off) and section 2.3
// / Fig. 3 (block-wise scales set by the block maximum); formats from the
// feature list (MXFP4 / NVFP4).
//
// Per 128 x 128 tile of A (one CTA, 128 threads):
//   1. TMA loads the tile's rows of U (hi, lo) and of W = V diag(S) (hi, lo),
//      bf16, K = k padded to 64 (zeros).
//   2. One thread issues U_hi W_hi + U_hi W_lo + U_lo W_hi as kind::f16 MMAs
//      into a 128 x 128 fp32 TMEM accumulator: L = U S V^T to ~2^-16.
//   3. Every thread owns one row: for each 64-column chunk it reads L from
//      TMEM and A from global memory, forms R = fl32(a - l) and
//        amax pass:  keeps max |R| (NVFP4 needs the tensor maximum first),
//        quantize:   blocks along n straight from registers (32 bytes of
//                    codes per thread); blocks along m through a per-warp
//                    32 x 64 shared-memory transpose (a warp's 32 rows are
//                    one MXFP4 block or two NVFP4 blocks of every column);
//                    optional float32 tap of R.
// HBM-bound: A is read once per pass (twice for NVFP4) and FP4 codes plus
// scales are written once per quantized axis.
#include "abi_common.h"
#include "common.cuh"
#include "fp4_block.cuh"
#include "residual_quant.h"

namespace metis {

namespace {

constexpr int kTile = 128;

MDEV bool wait_ns(uint64_t* bar, uint32_t parity, uint64_t ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > ns) return false;
  }
  return true;
}

MDEV void load64(const void* A, int dtype, int64_t idx, int n, float* v) {
  if (dtype == METIS_BF16) {
    const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(A) + idx);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (8 * q < n) {
        const uint4 u = p[q];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[8 * q + 2 * i] = __uint_as_float(w[i] << 16);
          v[8 * q + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
      }
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(A) + idx);
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      if (4 * q < n) {
        const float4 f = p[q];
        v[4 * q] = f.x;
        v[4 * q + 1] = f.y;
        v[4 * q + 2] = f.z;
        v[4 * q + 3] = f.w;
      }
    }
  }
}

// Quantize n (32 or 64) values along the block axis: outer index o, first
// element at inner offset i0 (a multiple of 32).
MDEV void emit(const float* v, int n, int fmt, float s_t, uint8_t* codes, uint8_t* scales, int64_t scale_cols,
               int64_t inner, int64_t o, int64_t i0) {
  uint8_t* dst = codes + o * (inner / 2) + i0 / 2;
  if (fmt == METIS_NVFP4) {
    uint64_t pk[4] = {0, 0, 0, 0};
    uint32_t sc = 0;
    const int nb = n / 16;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      if (b < nb) {
        float ds;
        sc |= quant_block_nv(v + 16 * b, s_t, pk[b], ds) << (8 * b);
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

__global__ void __launch_bounds__(128) residual_quant_kernel(const ResidualParams p,
                                                             const __grid_constant__ CUtensorMap tmUhi,
                                                             const __grid_constant__ CUtensorMap tmUlo,
                                                             const __grid_constant__ CUtensorMap tmWhi,
                                                             const __grid_constant__ CUtensorMap tmWlo) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int chunks = p.kp / 64;
  const int part = chunks * 16384;  // one operand part: 128 rows x kp bf16
  uint8_t* sUhi = smem;
  uint8_t* sUlo = sUhi + part;
  uint8_t* sWhi = sUlo + part;
  uint8_t* sWlo = sWhi + part;
  float* stage = reinterpret_cast<float*>(sWlo + part);  // 4 warps x 32 x 65 floats
  uint64_t* bars = reinterpret_cast<uint64_t*>(stage + 4 * 32 * 65);
  uint64_t* loaded = bars;
  uint64_t* done = bars + 1;
  uint32_t* tmem_sh = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_sh + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tn = blockIdx.x, tm = blockIdx.y;
  if (threadIdx.x == 0) {
    mbar_init(loaded, 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_sh, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_sh;

  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(loaded, 4 * part);
    for (int c = 0; c < chunks; ++c) {
      tma_load_2d(sUhi + c * 16384, &tmUhi, loaded, 64 * c, tm * kTile);
      tma_load_2d(sUlo + c * 16384, &tmUlo, loaded, 64 * c, tm * kTile);
      tma_load_2d(sWhi + c * 16384, &tmWhi, loaded, 64 * c, tn * kTile);
      tma_load_2d(sWlo + c * 16384, &tmWlo, loaded, 64 * c, tn * kTile);
    }
  } else if (threadIdx.x == 32) {
    if (mbar_wait(loaded, 0, abort_flag)) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16(128, kTile, false, false);
      uint32_t acc = 0;
      for (int c = 0; c < chunks; ++c) {
        const uint64_t uh = make_sdesc(smem_u32(sUhi + c * 16384), 16, 1024, kSwizzle128B);
        const uint64_t ul = make_sdesc(smem_u32(sUlo + c * 16384), 16, 1024, kSwizzle128B);
        const uint64_t wh = make_sdesc(smem_u32(sWhi + c * 16384), 16, 1024, kSwizzle128B);
        const uint64_t wl = make_sdesc(smem_u32(sWlo + c * 16384), 16, 1024, kSwizzle128B);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t o = static_cast<uint64_t>(2 * j);
          mma_bf16(tmem, uh + o, wh + o, idesc, acc);
          acc = 1;
          mma_bf16(tmem, uh + o, wl + o, idesc, 1);
          mma_bf16(tmem, ul + o, wh + o, idesc, 1);
        }
      }
    }
    tc_commit(done);
  }
  __syncwarp();
  const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(done, 0, abort_flag));
  tc_fence_after();

  float s_t = 1.f;
  if (p.mode == 1 && p.fmt == METIS_NVFP4) s_t = nv_tensor_scale(__uint_as_float(*p.amax_bits));
  if (p.mode == 1 && p.fmt == METIS_NVFP4 && tm == 0 && tn == 0 && threadIdx.x == 0) {
    if (p.ts_rows) *p.ts_rows = s_t;
    if (p.ts_cols) *p.ts_cols = s_t;
  }
  const int64_t row = static_cast<int64_t>(tm) * kTile + 32 * warp + lane;
  const bool row_ok = row < p.m;
  float amax = 0.f;
  float* my_stage = stage + warp * 32 * 65;
  for (int h = 0; h < 2; ++h) {
    const int64_t col0 = static_cast<int64_t>(tn) * kTile + 64 * h;
    const int ncols = static_cast<int>(imax64(0, imin64(64, p.n - col0)));  // 0, 32 or 64
    float v[64];
    uint32_t L[64];
    if (ok) {
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld16(tmem + (static_cast<uint32_t>(32 * warp) << 16) + 64 * h + 16 * q, L + 16 * q);
      tmem_ld_wait();
    }
    if (ncols == 0) continue;
    if (row_ok) load64(p.A, p.dtype, row * p.lda + col0, ncols, v);
#pragma unroll
    for (int j = 0; j < 64; ++j) {
      const float l = ok ? __uint_as_float(L[j]) : 0.f;
      v[j] = (row_ok && j < ncols) ? __fsub_rn(v[j], l) : 0.f;
    }
    if (p.mode == 0) {
#pragma unroll
      for (int j = 0; j < 64; ++j) amax = fmaxf(amax, fabsf(v[j]));
      continue;
    }
    if (row_ok && p.r_tap) {
      float* t = p.r_tap + row * p.n + col0;
      for (int j = 0; j < ncols; j += 4) *reinterpret_cast<float4*>(t + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
    }
    if (row_ok && p.r_codes) emit(v, ncols, p.fmt, s_t, p.r_codes, p.r_scales, p.r_scale_cols, p.n, row, col0);
    if (p.c_codes) {
      // transpose the warp's 32 rows x 64 columns through shared memory
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 64; ++j) my_stage[lane * 65 + j] = v[j];
      __syncwarp();
      const int64_t r0 = static_cast<int64_t>(tm) * kTile + 32 * warp;
      if (r0 < p.m) {
        for (int cc = 0; cc < 2; ++cc) {
          const int c = 2 * lane + cc;
          if (c < ncols) {
            float col[32];
#pragma unroll
            for (int r = 0; r < 32; ++r) col[r] = my_stage[r * 65 + c];
            emit(col, 32, p.fmt, s_t, p.c_codes, p.c_scales, p.c_scale_cols, p.m, col0 + c, r0);
          }
        }
      }
    }
  }
  if (p.mode == 0) {
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if (lane == 0) atomicMax(p.amax_bits, __float_as_uint(amax));
  }
  if (*abort_flag && threadIdx.x == 32) wait_ns(done, 0, 100000000ull);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
  if (threadIdx.x == 0 && *abort_flag) report(p.dev_status, METIS_DEV_TIMEOUT);
}

// U (rows x k) times diag(S) (optional) -> hi / lo bf16 [rows][kp], zero padded.
__global__ void hilo_kernel(const float* X, int64_t rows, int k, const float* S, int kp, __nv_bfloat16* hi,
                            __nv_bfloat16* lo) {
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < rows * kp;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = e / kp;
    const int c = static_cast<int>(e - r * kp);
    float x = 0.f;
    if (c < k) {
      x = X[r * k + c];
      if (S) x = __fmul_rn(x, S[c]);
    }
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    hi[e] = h;
    lo[e] = __float2bfloat16_rn(__fsub_rn(x, __bfloat162float(h)));
  }
}

CUresult map_rows(CUtensorMap* m, const void* base, int64_t rows, int kp) {
  const uint64_t dims[2] = {static_cast<uint64_t>(kp), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(kp) * 2};
  const uint32_t box[2] = {64, 128};
  return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

void launch_hilo(const float* X, int64_t rows, int k, const float* S, int kp, __nv_bfloat16* hi, __nv_bfloat16* lo,
                 int sms, cudaStream_t s) {
  int64_t b = (rows * kp + 255) / 256;
  if (b > sms * 8) b = sms * 8;
  hilo_kernel<<<static_cast<unsigned>(b < 1 ? 1 : b), 256, 0, s>>>(X, rows, k, S, kp, hi, lo);
}

metis_status run_residual_quant(const ResidualParams& p, const ResidualOperands& o, cudaStream_t s) {
  CUtensorMap uh, ul, wh, wl;
  if (map_rows(&uh, o.u_hi, p.m, p.kp) != CUDA_SUCCESS || map_rows(&ul, o.u_lo, p.m, p.kp) != CUDA_SUCCESS ||
      map_rows(&wh, o.w_hi, p.n, p.kp) != CUDA_SUCCESS || map_rows(&wl, o.w_lo, p.n, p.kp) != CUDA_SUCCESS)
    return fail(METIS_ERR_CUDA, "residual tensor map");
  const int part = (p.kp / 64) * 16384;
  const int smem = 4 * part + 4 * 32 * 65 * 4 + 64 + 1024;
  if (!ensure_smem(reinterpret_cast<const void*>(residual_quant_kernel), smem))
    return fail(METIS_ERR_CUDA, "residual shared-memory attribute");
  const dim3 grid(static_cast<unsigned>((p.n + kTile - 1) / kTile), static_cast<unsigned>((p.m + kTile - 1) / kTile));
  residual_quant_kernel<<<grid, 128, smem, s>>>(p, uh, ul, wh, wl);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(METIS_ERR_CUDA, "residual_quant launch", cudaGetErrorString(e));
  return METIS_OK;
}

}  // namespace metis
