// Tall-skinny bf16 GEMMs of the randomized range finder on tcgen05, with the
// split-K reduction and the consumers' outputs fused into the epilogue:
//   mode 0:  Y = A X      (m x lp), contraction over A's columns
//   mode 1:  Y = A^T X    (n x lp), contraction over A's rows
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
// Work split: one thread-block cluster of `cs` CTAs per 128-row output tile;
// CTA r of the cluster multiplies the r-th K slice into its own TMEM
// accumulator (128 threads: warp 0 lane 0 issues TMA, warp 1 lane 0 issues
// MMAs).  The epilogue (all four warps) stages the slice's partial tile in
// shared memory; the partial tiles are then summed through distributed shared
// memory in the fixed order r = 0, 1, ..., cs - 1 (so the result does not
// depend on timing), each CTA finishing 128 / cs rows.  A CTA writes its rows
// as float32 (optional) and as a transposed bf16 hi / lo copy (optional: the
// X operand of the next pass).  The float64 Gram of Y, where one is needed,
// is a separate many-CTA pass over the float32 rows (small_linalg.cu).
#include "abi_common.h"
#include "common.cuh"
#include "skinny_gemm.h"

namespace metis {

namespace {

constexpr int kStages = 3;
constexpr int kTileRows = 128;

MDEV bool wait_ns(uint64_t* bar, uint32_t parity, uint64_t ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > ns) return false;
  }
  return true;
}

struct SkinnySmem {
  int stage_bytes, ring, red, fin, epi, bars, total;
};

// Shared-memory plan: the TMA ring, then (aliasing it once the main loop is
// done) the partial tile `red` [128][lp + 4] floats and the finished rows
// `fin` [128 / cs][lp + 4] floats (the partial tile itself when cs = 1);
// barriers after the larger of the two.  Rows of lp + 4 floats keep 16-byte
// alignment for the vector copies and spread a warp's rows over the banks.
__host__ __device__ inline SkinnySmem skinny_smem(int aparts, int nmma, int lp, int cs) {
  SkinnySmem s{};
  const int ld = lp + 4;
  const int rs = kTileRows / cs;
  s.stage_bytes = ((aparts * 16384 + nmma * 128) + 1023) & ~1023;
  s.ring = kStages * s.stage_bytes;
  s.red = kTileRows * ld * 4;
  s.fin = cs == 1 ? 0 : rs * ld * 4;
  s.epi = s.red + s.fin;
  s.bars = ((s.ring > s.epi ? s.ring : s.epi) + 1023) & ~1023;
  s.total = s.bars + 256 + 1024;   // barriers, alignment slack
  return s;
}

__global__ void __launch_bounds__(128) skinny_gemm_kernel(const SkinnyParams p, const __grid_constant__ CUtensorMap tmA0,
                                                          const __grid_constant__ CUtensorMap tmA1,
                                                          const __grid_constant__ CUtensorMap tmX) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int cs = p.cs;
  const SkinnySmem L = skinny_smem(p.aparts, p.nmma, p.lp, cs);
  const int a_bytes = 16384;
  const int x_bytes = p.nmma * 128;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + kStages;
  uint64_t* done = empty + kStages;
  uint32_t* tmem_sh = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_sh + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x;
  const int rank = blockIdx.y;  // the K slice, = the CTA's rank in its cluster
  const int64_t ks0 = static_cast<int64_t>(rank) * p.ksteps_per_split;
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
      uint8_t* s = smem + stage * L.stage_bytes;
      const int32_t k0 = static_cast<int32_t>((ks0 + it) * 64);
      mbar_arrive_expect_tx(&full[stage], p.aparts * a_bytes + x_bytes);
      for (int a = 0; a < p.aparts; ++a) {
        const CUtensorMap* m = a == 0 ? &tmA0 : &tmA1;
        uint8_t* d = s + a * a_bytes;
        if (p.mode == 0) {
          tma_load_2d(d, m, &full[stage], k0, tile * kTileRows);
        } else {
          tma_load_2d(d, m, &full[stage], tile * kTileRows, k0);
          tma_load_2d(d + 8192, m, &full[stage], tile * kTileRows + 64, k0);
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
      uint8_t* s = smem + stage * L.stage_bytes;
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

  // ---- epilogue, all four warps: this slice's partial tile into `red`
  const int lp = p.lp;
  const int ld = lp + 4;
  const int lp4 = lp / 4;
  float* red = reinterpret_cast<float*>(smem);
  const bool have = nsteps > 0;
  bool ok = true;
  if (have) ok = mbar_wait(done, 0, abort_flag);
  tc_fence_after();
  {
    const int t = threadIdx.x;  // tile row = TMEM lane
    for (int c0 = 0; c0 < lp; c0 += 16) {
      uint32_t v[16], w[16];
      if (have && ok) {
        tmem_ld16(tmem + (static_cast<uint32_t>(32 * warp) << 16) + c0, v);
        if (p.xparts == 2) tmem_ld16(tmem + (static_cast<uint32_t>(32 * warp) << 16) + lp + c0, w);
        tmem_ld_wait();
      }
#pragma unroll
      for (int j = 0; j < 16; j += 4) {
        float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
        if (have && ok) {
          f = make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]), __uint_as_float(v[j + 2]),
                          __uint_as_float(v[j + 3]));
          if (p.xparts == 2) {
            f.x += __uint_as_float(w[j]);
            f.y += __uint_as_float(w[j + 1]);
            f.z += __uint_as_float(w[j + 2]);
            f.w += __uint_as_float(w[j + 3]);
          }
        }
        *reinterpret_cast<float4*>(red + t * ld + c0 + j) = f;
      }
    }
  }
  if (*abort_flag && warp == 1 && lane == 0) wait_ns(done, 0, 100000000ull);  // MMAs in flight
  tc_fence_before();
  if (cs > 1)
    cluster_sync_all();
  else
    __syncthreads();

  // ---- the cluster's sum for rows [r0, r0 + rs) of the tile, fixed order
  const int rs = kTileRows / cs;
  const int r0 = rank * rs;
  float* fin = cs == 1 ? red : reinterpret_cast<float*>(smem + L.red);
  if (cs > 1) {
    const uint32_t red_u32 = smem_u32(red);
    for (int e = threadIdx.x; e < rs * lp4; e += blockDim.x) {
      const int i = e / lp4, c = 4 * (e - i * lp4);
      const uint32_t off = static_cast<uint32_t>(((r0 + i) * ld + c) * 4);
      float4 part[8];
#pragma unroll
      for (int s = 0; s < 8; ++s)
        if (s < cs) part[s] = ld_cluster_f32x4(map_to_rank(red_u32 + off, static_cast<uint32_t>(s)));
      float4 sum = part[0];
#pragma unroll
      for (int s = 1; s < 8; ++s)
        if (s < cs) {
          sum.x += part[s].x;
          sum.y += part[s].y;
          sum.z += part[s].z;
          sum.w += part[s].w;
        }
      *reinterpret_cast<float4*>(fin + i * ld + c) = sum;
    }
    __syncthreads();
  }
  const int64_t grow0 = static_cast<int64_t>(tile) * kTileRows + r0;  // first global row of the slice
  const int nr = static_cast<int>(imax64(0, imin64(rs, p.rows_out - grow0)));
  if (p.out) {
    for (int e = threadIdx.x; e < nr * lp4; e += blockDim.x) {
      const int i = e / lp4, c = 4 * (e - i * lp4);
      *reinterpret_cast<float4*>(p.out + (grow0 + i) * lp + c) = *reinterpret_cast<const float4*>(fin + i * ld + c);
    }
  }
  if (p.outT) {  // row fastest: runs of consecutive rows of each column of Y^T
    for (int e = threadIdx.x; e < nr * lp; e += blockDim.x) {
      const int c = e / nr, i = e - c * nr;
      const float v = fin[i * ld + c];
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      p.outT[static_cast<int64_t>(c) * p.ldo + grow0 + i] = hi;
      p.outT[static_cast<int64_t>(lp + c) * p.ldo + grow0 + i] = __float2bfloat16_rn(__fsub_rn(v, __bfloat162float(hi)));
    }
  }
  // no CTA leaves while another may still read its shared memory
  if (cs > 1) cluster_sync_all();
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

int skinny_tiles(int64_t rows_out) { return static_cast<int>((rows_out + kTileRows - 1) / kTileRows); }

int skinny_cluster(int64_t rows_out, int64_t K, int sms) {
  const int64_t tiles = skinny_tiles(rows_out);
  const int64_t ksteps = (K + 63) / 64;
  // two CTAs fit on an SM: fill that one wave, in clusters of 1, 2, 4 or 8
  // CTAs, each with at least two K steps
  int cs = 1;
  while (cs < 8 && tiles * cs * 2 <= 2 * static_cast<int64_t>(sms) && ksteps >= 4 * cs) cs *= 2;
  return cs;
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
  p.cs = c.cs;
  p.ksteps_per_split = (p.total_ksteps + c.cs - 1) / c.cs;
  p.out = c.out;
  p.outT = c.outT;
  p.ldo = c.ldo;
  p.dev_status = c.dev_status;
  if (p.nmma % 16 || p.nmma > 256 || p.lp % 16) return METIS_ERR_ARG;
  if (c.cs != 1 && c.cs != 2 && c.cs != 4 && c.cs != 8) return METIS_ERR_ARG;
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
  const SkinnySmem L = skinny_smem(c.aparts, p.nmma, p.lp, c.cs);
  const void* fn = reinterpret_cast<const void*>(skinny_gemm_kernel);
  if (!ensure_smem(fn, L.total)) return fail(METIS_ERR_CUDA, "skinny_gemm shared-memory attribute");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(skinny_tiles(p.rows_out)), static_cast<unsigned>(c.cs));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = static_cast<size_t>(L.total);
  cfg.stream = s;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 1;
  attr.val.clusterDim.y = static_cast<unsigned>(c.cs);
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, skinny_gemm_kernel, p, ma0, ma1, mx);
  if (e != cudaSuccess) return fail(METIS_ERR_CUDA, "skinny_gemm launch", cudaGetErrorString(e));
  return METIS_OK;
}

}  // namespace metis
