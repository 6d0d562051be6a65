// Tall-skinny bf16 GEMMs of the randomized range finder on tcgen05:
//   mode 0:  P[s] = A X      (m x lp), contraction over A's columns
//   mode 1:  P[s] = A^T X    (n x lp), contraction over A's rows
// with split-K partial sums P[s] (s = 0..splits-1, summed later in a fixed
// order, so results are deterministic).
//
// Source: SII release on Metis, section 2.4 item 1 (randomized dimension
// reduction: the decomposition runs on a low-dimensional sketch); "Metis:
// Training LLMs with FP4 Quantization" technical framework (random
// projection).  Y = A Omega, the power iteration A^T Q / A Q and the core
// projection B^T = A^T Q are all one pass over A each.
//
// HBM-bound: the l <= 128 sketch columns give ~l flop per byte of A, far
// below the bf16 ridge, so the kernel streams A once with TMA (A K-major for
// mode 0; MN-major, two 64-column boxes, for mode 1) and issues one MMA of
// N = parts * lp per 16-deep K step.  X holds up to two bf16 parts (hi, lo
// of an fp32 operand) stacked as rows [0, lp) and [lp, 2 lp) of X^T, so one
// MMA computes both products; the epilogue adds them.  An fp32 A is given as
// two bf16 parts (hi, lo) that accumulate into the same TMEM accumulator.
//
// One CTA per (128-row output tile, K split), 128 threads: warp 0 lane 0
// issues TMA, warp 1 lane 0 issues MMAs, all four warps drain TMEM.
#include "abi_common.h"
#include "common.cuh"
#include "skinny_gemm.h"

namespace metis {

namespace {

constexpr int kStages = 3;

MDEV bool wait_ns(uint64_t* bar, uint32_t parity, uint64_t ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > ns) return false;
  }
  return true;
}

__global__ void __launch_bounds__(128) skinny_gemm_kernel(const SkinnyParams p, const __grid_constant__ CUtensorMap tmA0,
                                                          const __grid_constant__ CUtensorMap tmA1,
                                                          const __grid_constant__ CUtensorMap tmX) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int a_bytes = 16384;
  const int x_bytes = p.nmma * 128;
  const int stage_bytes = ((p.aparts * a_bytes + x_bytes) + 1023) & ~1023;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * stage_bytes);
  uint64_t* empty = full + kStages;
  uint64_t* done = empty + kStages;
  uint32_t* tmem_sh = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_sh + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, split = blockIdx.y;
  const int64_t ks0 = static_cast<int64_t>(split) * p.ksteps_per_split;
  int64_t ks1 = ks0 + p.ksteps_per_split;
  if (ks1 > p.total_ksteps) ks1 = p.total_ksteps;
  const int nsteps = ks1 > ks0 ? static_cast<int>(ks1 - ks0) : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_sh, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_sh;

  if (warp == 0 && lane == 0 && nsteps > 0) {
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    for (int it = 0; it < nsteps; ++it) {
      if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) break;
      uint8_t* s = smem + stage * stage_bytes;
      const int32_t k0 = static_cast<int32_t>((ks0 + it) * 64);
      mbar_arrive_expect_tx(&full[stage], p.aparts * a_bytes + x_bytes);
      for (int a = 0; a < p.aparts; ++a) {
        const CUtensorMap* m = a == 0 ? &tmA0 : &tmA1;
        uint8_t* d = s + a * a_bytes;
        if (p.mode == 0) {
          tma_load_2d(d, m, &full[stage], k0, tile * 128);
        } else {
          tma_load_2d(d, m, &full[stage], tile * 128, k0);
          tma_load_2d(d + 8192, m, &full[stage], tile * 128 + 64, k0);
        }
      }
      tma_load_2d(s + p.aparts * a_bytes, &tmX, &full[stage], k0, 0);
      ++issued;
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (*abort_flag) {
      int s = stage;
      uint32_t ph = phase;
      for (int i = 0; i < min(issued, kStages); ++i) {
        if (--s < 0) {
          s = kStages - 1;
          ph ^= 1u;
        }
        wait_ns(&full[s], ph, 100000000ull);
      }
    }
  } else if (warp == 1 && lane == 0) {
    int stage = 0;
    uint32_t phase = 0;
    uint32_t acc = 0;
    const uint32_t idesc = idesc_bf16(128, p.nmma, p.mode == 1, false);
    bool ok = true;
    for (int it = 0; it < nsteps; ++it) {
      if (!mbar_wait(&full[stage], phase, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint8_t* s = smem + stage * stage_bytes;
      const uint64_t xdesc = make_sdesc(smem_u32(s + p.aparts * a_bytes), 16, 1024, kSwizzle128B);
      for (int a = 0; a < p.aparts; ++a) {
        const uint32_t sa = smem_u32(s + a * a_bytes);
        const uint64_t adesc = p.mode == 0 ? make_sdesc(sa, 16, 1024, kSwizzle128B)
                                           : make_sdesc(sa, 8192, 1024, kSwizzle128B);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t aoff = p.mode == 0 ? static_cast<uint64_t>(2 * j) : static_cast<uint64_t>(128 * j);
          mma_bf16(tmem, adesc + aoff, xdesc + static_cast<uint64_t>(2 * j), idesc, acc);
          acc = 1;
        }
      }
      tc_commit(&empty[stage]);
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    tc_commit(done);
    if (!ok) report(p.dev_status, METIS_DEV_TIMEOUT);
  }
  __syncwarp();

  // epilogue: all four warps, one output row per thread
  const bool have = nsteps > 0;
  bool ok = true;
  if (have) ok = mbar_wait(done, 0, abort_flag);
  tc_fence_after();
  const int64_t row = static_cast<int64_t>(tile) * 128 + 32 * warp + lane;
  float* dst = p.out + (static_cast<int64_t>(split) * p.rows_out + row) * p.lp;
  for (int c0 = 0; c0 < p.lp; c0 += 16) {
    uint32_t v[16], w[16];
    if (have && ok) {
      tmem_ld16(tmem + (static_cast<uint32_t>(32 * warp) << 16) + c0, v);
      if (p.xparts == 2) tmem_ld16(tmem + (static_cast<uint32_t>(32 * warp) << 16) + p.lp + c0, w);
      tmem_ld_wait();
    }
    if (row < p.rows_out) {
#pragma unroll
      for (int j = 0; j < 16; j += 4) {
        float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
        if (have && ok) {
          f.x = __uint_as_float(v[j]);
          f.y = __uint_as_float(v[j + 1]);
          f.z = __uint_as_float(v[j + 2]);
          f.w = __uint_as_float(v[j + 3]);
          if (p.xparts == 2) {
            f.x += __uint_as_float(w[j]);
            f.y += __uint_as_float(w[j + 1]);
            f.z += __uint_as_float(w[j + 2]);
            f.w += __uint_as_float(w[j + 3]);
          }
        }
        *reinterpret_cast<float4*>(dst + c0 + j) = f;
      }
    }
  }
  if (*abort_flag && warp == 1 && lane == 0) wait_ns(done, 0, 100000000ull);  // MMAs in flight
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
  if (threadIdx.x == 0 && *abort_flag) report(p.dev_status, METIS_DEV_TIMEOUT);
}

CUresult map_bf16(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld, uint32_t box_cols,
                  uint32_t box_rows) {
  const uint64_t dims[2] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(ld) * 2};
  const uint32_t box[2] = {box_cols, box_rows};
  return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

int skinny_splits(int64_t rows_out, int64_t K, int sms) {
  const int64_t tiles = (rows_out + 127) / 128;
  const int64_t ksteps = (K + 63) / 64;
  // two CTAs fit on an SM: fill that one wave without starting a second
  int64_t s = 2 * static_cast<int64_t>(sms) / tiles;
  if (s > ksteps) s = ksteps;
  if (s < 1) s = 1;
  return static_cast<int>(s);
}

metis_status run_skinny_gemm(const SkinnyCall& c, cudaStream_t s) {
  SkinnyParams p{};
  p.mode = c.mode;
  p.rows_out = c.mode == 0 ? c.m : c.n;
  p.K = c.mode == 0 ? c.n : c.m;
  p.lp = c.lp;
  p.xparts = c.xparts;
  p.aparts = c.aparts;
  p.nmma = c.lp * c.xparts;
  p.total_ksteps = (p.K + 63) / 64;
  p.splits = c.splits;
  p.ksteps_per_split = (p.total_ksteps + c.splits - 1) / c.splits;
  p.out = c.out;
  p.dev_status = c.dev_status;
  if (p.nmma % 16 || p.nmma > 256 || p.lp % 16) return METIS_ERR_ARG;
  CUtensorMap ma0, ma1, mx;
  for (int a = 0; a < c.aparts; ++a) {
    CUtensorMap* m = a == 0 ? &ma0 : &ma1;
    const CUresult r = c.mode == 0 ? map_bf16(m, c.A[a], c.m, c.n, c.lda, 64, 128)
                                    : map_bf16(m, c.A[a], c.m, c.n, c.lda, 64, 64);
    if (r != CUDA_SUCCESS) return fail(METIS_ERR_CUDA, "skinny_gemm tensor map");
  }
  if (c.aparts == 1) ma1 = ma0;
  if (map_bf16(&mx, c.Xt, p.nmma, p.K, c.ldx, 64, static_cast<uint32_t>(p.nmma)) != CUDA_SUCCESS)
    return fail(METIS_ERR_CUDA, "skinny_gemm tensor map");
  const int stage_bytes = ((c.aparts * 16384 + p.nmma * 128) + 1023) & ~1023;
  const int smem = kStages * stage_bytes + 1024 + 256;
  if (!ensure_smem(reinterpret_cast<const void*>(skinny_gemm_kernel), smem))
    return fail(METIS_ERR_CUDA, "skinny_gemm shared-memory attribute");
  const dim3 grid(static_cast<unsigned>((p.rows_out + 127) / 128), static_cast<unsigned>(c.splits));
  skinny_gemm_kernel<<<grid, 128, smem, s>>>(p, ma0, ma1, mx);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(METIS_ERR_CUDA, "skinny_gemm launch", cudaGetErrorString(e));
  return METIS_OK;
}

}  // namespace metis
