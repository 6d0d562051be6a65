// Block-scaled FP4 GEMM on the sm_100a tensor cores (tcgen05), with an
// optional low-rank update accumulated into the same TMEM accumulator.
//
// Source: "Metis: Training LLMs with FP4 Quantization" abstract (W4A4G4: the
// forward and both backward products run on FP4 operands); SII release
// section 2.4 item 1 (the dominant low-rank part and the long-tail residual
// both enter the product).
//
//   C[M x N] = alpha * ( sum_k A_q[m,k] B_q[n,k]  (FP4, block scales applied
//                                                  by the MMA)
//                        + sum_j LA[m,j] LB[n,j] ) (bf16 low-rank chunks)
//
// A_q, B_q: FP4 codes, K-major ([rows][K/2] bytes) with the tensor-core scale
// layout; alpha = product of the NVFP4 tensor scales (1 for MXFP4).
//
// Design (one persistent CTA per SM, 352 threads, warp-specialized):
//   warp 0      TMA producer: per 256-element K tile loads the A tile
//               (128 rows x 128 B) and B tile (BN rows x 128 B) with 128-byte
//               swizzle (completing on the stage's operand barrier), and the
//               matching 512-byte scale chunks with bulk copies (completing
//               on the stage's scale barrier, armed only for FP4 steps), into
//               a 4-stage shared-memory ring.
//   warp 1      TMEM allocator + MMA issuer: waits for a stage's operands and
//               its scale factors, issues four K=64 block-scaled MMAs
//               (kind::mxf4 / mxf4nvf4), then kind::f16 MMAs for the low-rank
//               chunks, and commits.
//   warps 2-9   epilogue: drain the 128 x BN fp32 accumulator from TMEM into
//               registers, release it, scale and store (fp32 or bf16), or
//               store raw partial sums for split-K.
//   warp 10     scale copies: waits for a stage's scale chunks, copies them
//               into that stage's own TMEM columns (tcgen05.cp
//               32x128b.warpx4) and commits them to a per-stage barrier the
//               MMA warp waits on; issued by the MMA warp itself, the copies
//               sat in front of every stage's MMAs (125.7 against 105.3 us on
//               8192 x 4096 x 4096 NVFP4).  Both scale barriers count FP4
//               steps only, so the low-rank steps the scale warp skips never
//               let a parity wait pass a phase early.
// Every wait is bounded (METIS_DEV_TIMEOUT) and the kernel always frees its
// TMEM.  Shared memory per stage: A 16 KB + B BN*128 B + scales 6 KB.
//
// A second kernel, gemm_fp4_wide_kernel, runs the same pipeline (scale warp
// included) on a 256 x 192 tile (two 128-row M halves sharing one B tile,
// three stages, two TMEM scale slots);
// run_gemm_fp4 picks it for unsplit products when its rounds of tiles over
// the SMs cost less than the 128 x 256 tile's.
#include "abi_common.h"
#include "common.cuh"
#include "gemm_fp4.h"

namespace metis {

namespace {

// warps 0-1 producer and MMA issuer, 2-9 epilogue, 10 the scale copies
constexpr int kSfWarp = 10;
constexpr int kThreads = 32 * (kSfWarp + 1);
constexpr int kEpiWarps = 8;

template <int BN, int STAGES>
struct Smem {
  static constexpr int kA = 128 * 128;
  static constexpr int kB = BN * 128;
  static constexpr int kSFA = 2048;
  static constexpr int kSFB = BN > 128 ? 4096 : 2048;
  static constexpr int kStage = kA + kB + kSFA + kSFB;
  static constexpr int kBytes = STAGES * kStage + 1024 /*align*/ + 256 /*barriers*/;
};

MDEV bool wait_ns(uint64_t* bar, uint32_t parity, uint64_t ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > ns) return false;
  }
  return true;
}

// BN: MMA N; STAGES: shared-memory ring depth; CTAS: CTAs per SM (2 halves
// the TMEM allocation and lets one CTA's epilogue overlap the other's MMAs).
template <int BN, int STAGES, int CTAS>
__global__ void __launch_bounds__(kThreads, CTAS)
    gemm_fp4_kernel(const GemmParams p, const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmLA,
                    const __grid_constant__ CUtensorMap tmLB) {
  using S = Smem<BN, STAGES>;
  constexpr int kStages = STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * S::kStage);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* sf_ready = acc_empty + 1;   // per stage: its scale factors are in TMEM
  uint64_t* sf_full = sf_ready + kStages;  // per stage: its scale bytes are in shared memory
  uint32_t* tmem_base_sh = reinterpret_cast<uint32_t*>(sf_full + kStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_sh + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool nv = p.fmt == METIS_NVFP4;
  const int atoms_per_kt = nv ? 4 : 2;           // 512-byte scale chunks per 128 rows per K tile
  const int sfa_cols = 4 * atoms_per_kt;          // TMEM columns for A scales per stage
  constexpr int kBHalves = BN > 128 ? 2 : 1;      // 128-row scale chunk groups of B
  const int sfb_cols = 4 * atoms_per_kt * kBHalves;
  const int sf_stage_cols = sfa_cols + sfb_cols;
  constexpr uint32_t kTmemCols = CTAS == 2 ? 256 : 512;
  constexpr uint32_t kSfBase = CTAS == 2 ? BN : 256;  // TMEM columns of the accumulator

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_ready[s], 1);
      mbar_init(&sf_full[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEpiWarps);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    if (p.lr_chunks) {
      prefetch_tensormap(&tmLA);
      prefetch_tensormap(&tmLB);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_sh;

  const int tiles_m = (p.M + 127) / 128;
  const int tiles_n = (p.N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n * p.splits;
  const int kt_per_split = (p.num_kt + p.splits - 1) / p.splits;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      uint32_t sf_phase = 0;   // bit s: parity of sf_full[s]'s next phase
      uint32_t sf_last = 0;    // bit s: the last load into stage s carried scales
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const int split = t % p.splits;
        const int tt = t / p.splits;
        const int tm = tt % tiles_m;
        const int tn = tt / tiles_m;
        const int kt0 = split * kt_per_split;
        const int kt1 = min(p.num_kt, kt0 + kt_per_split);
        const int nlr = (split == p.splits - 1) ? p.lr_chunks : 0;
        for (int it = kt0; it < kt1 + nlr; ++it) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          uint8_t* sA = smem + stage * S::kStage;
          uint8_t* sB = sA + S::kA;
          uint8_t* sSFA = sB + S::kB;
          uint8_t* sSFB = sSFA + S::kSFA;
          if (it < kt1) {
            const int kt = it;
            const uint32_t sf_bytes = 512u * atoms_per_kt;
            const bool second = kBHalves == 2 && (2 * tn + 1) * 128 < p.sfb_rows;
            // the operands complete on full[stage] (MMA warp), the scale
            // chunks on sf_full[stage] (scale warp), which is armed only
            // for FP4 steps, so its phases count exactly the steps the scale
            // warp serves
            const uint32_t sbytes = sf_bytes * (1 + (kBHalves == 2 ? (second ? 2 : 1) : 1));
            mbar_arrive_expect_tx(&full[stage], S::kA + S::kB);
            mbar_arrive_expect_tx(&sf_full[stage], sbytes);
            tma_load_2d(sA, &tmA, &full[stage], kt * 128, tm * 128);
            tma_load_2d(sB, &tmB, &full[stage], kt * 128, tn * BN);
            bulk_load(sSFA, p.sfa + (static_cast<int64_t>(tm) * p.sfa_chunks + kt * atoms_per_kt) * 512,
                      sf_bytes, &sf_full[stage]);
            const int nb0 = kBHalves == 2 ? 2 * tn : tn * BN / 128;
            bulk_load(sSFB, p.sfb + (static_cast<int64_t>(nb0) * p.sfb_chunks + kt * atoms_per_kt) * 512,
                      sf_bytes, &sf_full[stage]);
            if (kBHalves == 2 && second)
              bulk_load(sSFB + 2048, p.sfb + (static_cast<int64_t>(nb0 + 1) * p.sfb_chunks + kt * atoms_per_kt) * 512,
                        sf_bytes, &sf_full[stage]);
            sf_phase ^= 1u << stage;
            sf_last |= 1u << stage;
          } else {
            const int c = it - kt1;
            mbar_arrive_expect_tx(&full[stage], S::kA + S::kB);
            tma_load_2d(sA, &tmLA, &full[stage], c * 64, tm * 128);
            tma_load_2d(sB, &tmLB, &full[stage], c * 64, tn * BN);
            sf_last &= ~(1u << stage);
          }
          ++issued;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (*abort_flag) {
        // let copies already in flight land before the CTA exits
        int s = stage;
        uint32_t ph = phase;
        for (int i = 0; i < min(issued, kStages); ++i) {
          if (--s < 0) { s = kStages - 1; ph ^= 1u; }
          wait_ns(&full[s], ph, 100000000ull);
          // sf_phase holds the parity after the last arming: the phase in
          // flight has the other one
          if ((sf_last >> s) & 1u) wait_ns(&sf_full[s], ((sf_phase >> s) & 1u) ^ 1u, 100000000ull);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_phase = 0;
      uint32_t sf_phase = 0;   // bit s: parity of sf_ready[s]'s next phase
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const int split = t % p.splits;
        const int tn = (t / p.splits) / tiles_m;
        // with BN = 64 a tile covers half of a 128-row scale chunk: the upper
        // half's scales sit two TMEM columns further
        const uint32_t sfb_off = BN == 64 ? 2u * (tn & 1) : 0u;
        const int kt0 = split * kt_per_split;
        const int kt1 = min(p.num_kt, kt0 + kt_per_split);
        const int nlr = (split == p.splits - 1) ? p.lr_chunks : 0;
        if (!mbar_wait(acc_empty, acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        uint32_t accumulate = 0;
        for (int it = kt0; it < kt1 + nlr; ++it) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
          // an FP4 stage's scale factors are copied into TMEM by the scale
          // warp; sf_ready[s] completes once per FP4 use of stage s (the
          // low-rank chunks have none), so its parity is kept per stage
          if (it < kt1) {
            if (!mbar_wait(&sf_ready[stage], (sf_phase >> stage) & 1u, abort_flag)) { ok = false; break; }
            sf_phase ^= 1u << stage;
          }
          tc_fence_after();
          uint8_t* sA = smem + stage * S::kStage;
          uint8_t* sB = sA + S::kA;
          const uint64_t adesc = make_sdesc(smem_u32(sA), 16, 1024, kSwizzle128B);
          const uint64_t bdesc = make_sdesc(smem_u32(sB), 16, 1024, kSwizzle128B);
          if (it < kt1) {
            const uint32_t sfa_t = tmem + kSfBase + stage * sf_stage_cols;
            const uint32_t sfb_t = sfa_t + sfa_cols + sfb_off;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint64_t koff = static_cast<uint64_t>((j * 32) >> 4);
              if (nv) {
                mma_nvf4(tmem, adesc + koff, bdesc + koff, idesc_fp4(128, BN, false, 0, 0),
                         sfa_t + 4 * j, sfb_t + 4 * kBHalves * j, accumulate);
              } else {
                const uint32_t id = 2u * (j & 1);
                mma_mxf4(tmem, adesc + koff, bdesc + koff, idesc_fp4(128, BN, true, id, id),
                         (sfa_t + 4 * (j >> 1)) | (id << 30), (sfb_t + 4 * kBHalves * (j >> 1)) | (id << 30),
                         accumulate);
              }
              accumulate = 1;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint64_t koff = static_cast<uint64_t>((j * 32) >> 4);
              mma_bf16(tmem, adesc + koff, bdesc + koff, idesc_bf16(128, BN, false, false), accumulate);
              accumulate = 1;
            }
          }
          tc_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(acc_full);
        acc_phase ^= 1u;
      }
      if (*abort_flag) {
        // wait for MMAs already issued before the TMEM is freed
        tc_commit(acc_full);
        wait_ns(acc_full, acc_phase, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp == kSfWarp) {
    // ------------------------------------------------------------ scale copies
    // Each FP4 stage's scale factors go from shared memory into that stage's
    // own TMEM columns (tcgen05.cp 32x128b.warpx4), committed to sf_ready;
    // the MMA issuer waits for them, so copies of later stages are issued
    // while the MMAs of earlier ones run.  A stage's columns are rewritten
    // only after its smem was refilled, i.e. after the MMAs that read the
    // previous contents completed.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int last = -1;
      uint32_t last_phase = 0;
      uint32_t sf_phase = 0;   // bit s: parity of sf_ready[s]'s and sf_full[s]'s next phase
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const int split = t % p.splits;
        const int tn = (t / p.splits) / tiles_m;
        const uint32_t sfb_off = BN == 64 ? 2u * (tn & 1) : 0u;
        const int kt0 = split * kt_per_split;
        const int kt1 = min(p.num_kt, kt0 + kt_per_split);
        const int nlr = (split == p.splits - 1) ? p.lr_chunks : 0;
        for (int it = kt0; it < kt1 + nlr; ++it) {
          if (it < kt1) {
            if (!mbar_wait(&sf_full[stage], (sf_phase >> stage) & 1u, abort_flag)) { ok = false; break; }
            tc_fence_after();
            uint8_t* sSFA = smem + stage * S::kStage + S::kA + S::kB;
            uint8_t* sSFB = sSFA + S::kSFA;
            const uint32_t sfa_t = tmem + kSfBase + stage * sf_stage_cols;
            const uint32_t sfb_t = sfa_t + sfa_cols + sfb_off;
            for (int a = 0; a < atoms_per_kt; ++a) {
              tc_cp_32x128b_warpx4(sfa_t + 4 * a, make_sdesc(smem_u32(sSFA + 512 * a), 0, 128, kSwizzleNone));
              for (int h = 0; h < kBHalves; ++h)
                tc_cp_32x128b_warpx4(sfb_t - sfb_off + 4 * kBHalves * a + 4 * h,
                                     make_sdesc(smem_u32(sSFB + 2048 * h + 512 * a), 0, 128, kSwizzleNone));
            }
            tc_commit(&sf_ready[stage]);
            last = stage;
            last_phase = (sf_phase >> stage) & 1u;
            sf_phase ^= 1u << stage;
          }
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      // copies still in flight land before the TMEM is freed
      if (last >= 0) wait_ns(&sf_ready[last], last_phase, 100000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lane quadrant of this warp
    const int half = (warp - 2) >> 2;       // which BN/2 columns
    constexpr int kCols = BN / 2;           // columns per thread
    float alpha = 1.f;
    if (p.ts_a) alpha = __fmul_rn(alpha, *p.ts_a);
    if (p.ts_b) alpha = __fmul_rn(alpha, *p.ts_b);
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      const int split = t % p.splits;
      const int tt = t / p.splits;
      const int tm = tt % tiles_m;
      const int tn = tt / tiles_m;
      if (!mbar_wait(acc_full, acc_phase, abort_flag)) break;
      tc_fence_after();
      uint32_t v[kCols];
#pragma unroll
      for (int c = 0; c < kCols / 16; ++c)
        tmem_ld16(tmem + (static_cast<uint32_t>(32 * q) << 16) + half * kCols + 16 * c, v + 16 * c);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      acc_phase ^= 1u;
      const int64_t row = static_cast<int64_t>(tm) * 128 + 32 * q + lane;
      const int64_t col0 = static_cast<int64_t>(tn) * BN + half * kCols;
      if (row >= p.M) continue;
      if (p.partial) {
        float* dst = p.partial + (static_cast<int64_t>(split) * p.M + row) * p.N;
#pragma unroll
        for (int c = 0; c < kCols; c += 4) {
          const int64_t col = col0 + c;
          if (col + 3 < p.N && (p.N & 3) == 0) {
            *reinterpret_cast<float4*>(dst + col) = make_float4(__uint_as_float(v[c]), __uint_as_float(v[c + 1]),
                                                                __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
          } else {
            for (int e = 0; e < 4; ++e)
              if (col + e < p.N) dst[col + e] = __uint_as_float(v[c + e]);
          }
        }
      } else if (p.c_dtype == METIS_F32) {
        float* dst = reinterpret_cast<float*>(p.C) + row * p.ldc;
#pragma unroll
        for (int c = 0; c < kCols; c += 4) {
          const int64_t col = col0 + c;
          const float4 f = make_float4(__fmul_rn(alpha, __uint_as_float(v[c])), __fmul_rn(alpha, __uint_as_float(v[c + 1])),
                                       __fmul_rn(alpha, __uint_as_float(v[c + 2])), __fmul_rn(alpha, __uint_as_float(v[c + 3])));
          if (col + 3 < p.N && p.vec_ok) {
            *reinterpret_cast<float4*>(dst + col) = f;
          } else {
            const float fe[4] = {f.x, f.y, f.z, f.w};
            for (int e = 0; e < 4; ++e)
              if (col + e < p.N) dst[col + e] = fe[e];
          }
        }
      } else {
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.C) + row * p.ldc;
#pragma unroll
        for (int c = 0; c < kCols; c += 4) {
          const int64_t col = col0 + c;
          __nv_bfloat16 b[4];
          for (int e = 0; e < 4; ++e) b[e] = __float2bfloat16_rn(__fmul_rn(alpha, __uint_as_float(v[c + e])));
          if (col + 3 < p.N && p.vec_ok) {
            uint2 u;
            u.x = static_cast<uint32_t>(__bfloat16_as_ushort(b[0])) | (static_cast<uint32_t>(__bfloat16_as_ushort(b[1])) << 16);
            u.y = static_cast<uint32_t>(__bfloat16_as_ushort(b[2])) | (static_cast<uint32_t>(__bfloat16_as_ushort(b[3])) << 16);
            *reinterpret_cast<uint2*>(dst + col) = u;
          } else {
            for (int e = 0; e < 4; ++e)
              if (col + e < p.N) dst[col + e] = b[e];
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && *abort_flag) report(p.dev_status, METIS_DEV_TIMEOUT);
}

// ---------------------------------------------------------------------------
// Wide tile: two 128-row M halves share one 192-row B tile (256 x 192 per
// CTA).  Per flop it moves 22 % fewer operand bytes from L2 than a 128 x 256
// tile and issues fewer scale copies.  TMEM: the two halves' accumulators in
// columns 0-383 and the scale factors in two 64-column slots; the scale warp
// refills a slot only after the commit of the K step that last read it.  B's scale
// chunks come from the 128-row chunk at or below the tile's first row: a tile
// that starts 64 rows into a chunk (odd tn) reads them two TMEM columns
// further.  Rows past M and columns past N are computed on zero-filled (TMA)
// operands and never stored.  No split-K.
constexpr int kWideBN = 192;
constexpr int kWideStages = 3;
struct WideSmem {
  static constexpr int kA = 128 * 128;         // one M half, K = 256 FP4
  static constexpr int kB = kWideBN * 128;
  static constexpr int kSFA = 2048;            // per half
  static constexpr int kSFB = 4096;            // two 128-row chunks
  static constexpr int kStage = 2 * kA + kB + 2 * kSFA + kSFB;
  static constexpr int kBytes = kWideStages * kStage + 1024 /*align*/ + 256 /*barriers*/;
};

__global__ void __launch_bounds__(kThreads, 1)
    gemm_fp4_wide_kernel(const GemmParams p, const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmLA,
                         const __grid_constant__ CUtensorMap tmLB) {
  using S = WideSmem;
  constexpr int kStages = kWideStages;
  constexpr int BN = kWideBN;
  constexpr uint32_t kSfBase = 2 * BN;   // first TMEM column after the accumulators
  constexpr uint32_t kSlotCols = 64;     // per slot: A scales 2 x 16, B scales 32
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * S::kStage);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* sf_free = acc_empty + 1;     // [2]: the MMAs that read a slot have retired
  uint64_t* sf_ready = sf_free + 2;      // [2]: a slot holds the next K step's scales
  uint64_t* sf_full = sf_ready + 2;      // per stage: its scale bytes are in shared memory
  uint32_t* tmem_base_sh = reinterpret_cast<uint32_t*>(sf_full + kStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_sh + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool nv = p.fmt == METIS_NVFP4;
  const int atoms_per_kt = nv ? 4 : 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEpiWarps);
    mbar_init(&sf_free[0], 1);
    mbar_init(&sf_free[1], 1);
    mbar_init(&sf_ready[0], 1);
    mbar_init(&sf_ready[1], 1);
    for (int s = 0; s < kStages; ++s) mbar_init(&sf_full[s], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    if (p.lr_chunks) {
      prefetch_tensormap(&tmLA);
      prefetch_tensormap(&tmLB);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_sh, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_sh;

  const int tiles_m = (p.M + 255) / 256;
  const int tiles_n = (p.N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int nk = p.num_kt + p.lr_chunks;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      uint32_t sf_phase = 0;   // bit s: parity of sf_full[s]'s next phase
      uint32_t sf_last = 0;    // bit s: the last load into stage s carried scales
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const int tm = t % tiles_m, tn = t / tiles_m;
        const bool half1 = 256 * tm + 128 < p.M;               // A scales of the second half exist
        const int nb0 = tn * BN / 128;                         // B scale chunk at or below the tile
        const bool second = (nb0 + 1) * 128 < p.sfb_rows;
        for (int it = 0; it < nk; ++it) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          uint8_t* sA0 = smem + stage * S::kStage;
          uint8_t* sA1 = sA0 + S::kA;
          uint8_t* sB = sA1 + S::kA;
          uint8_t* sSFA0 = sB + S::kB;
          uint8_t* sSFA1 = sSFA0 + S::kSFA;
          uint8_t* sSFB = sSFA1 + S::kSFA;
          if (it < p.num_kt) {
            const int kt = it;
            const uint32_t sf_bytes = 512u * atoms_per_kt;
            // operands on full[stage] (MMA warp), scale chunks on sf_full[stage]
            // (scale warp), armed only for FP4 steps
            const uint32_t sbytes = sf_bytes * ((half1 ? 2 : 1) + (second ? 2 : 1));
            mbar_arrive_expect_tx(&full[stage], 2 * S::kA + S::kB);
            mbar_arrive_expect_tx(&sf_full[stage], sbytes);
            tma_load_2d(sA0, &tmA, &full[stage], kt * 128, 256 * tm);
            tma_load_2d(sA1, &tmA, &full[stage], kt * 128, 256 * tm + 128);
            tma_load_2d(sB, &tmB, &full[stage], kt * 128, tn * BN);
            bulk_load(sSFA0, p.sfa + (static_cast<int64_t>(2 * tm) * p.sfa_chunks + kt * atoms_per_kt) * 512, sf_bytes,
                      &sf_full[stage]);
            if (half1)
              bulk_load(sSFA1, p.sfa + (static_cast<int64_t>(2 * tm + 1) * p.sfa_chunks + kt * atoms_per_kt) * 512,
                        sf_bytes, &sf_full[stage]);
            bulk_load(sSFB, p.sfb + (static_cast<int64_t>(nb0) * p.sfb_chunks + kt * atoms_per_kt) * 512, sf_bytes,
                      &sf_full[stage]);
            if (second)
              bulk_load(sSFB + 2048, p.sfb + (static_cast<int64_t>(nb0 + 1) * p.sfb_chunks + kt * atoms_per_kt) * 512,
                        sf_bytes, &sf_full[stage]);
            sf_phase ^= 1u << stage;
            sf_last |= 1u << stage;
          } else {
            const int c = it - p.num_kt;
            mbar_arrive_expect_tx(&full[stage], 2 * S::kA + S::kB);
            tma_load_2d(sA0, &tmLA, &full[stage], c * 64, 256 * tm);
            tma_load_2d(sA1, &tmLA, &full[stage], c * 64, 256 * tm + 128);
            tma_load_2d(sB, &tmLB, &full[stage], c * 64, tn * BN);
            sf_last &= ~(1u << stage);
          }
          ++issued;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (*abort_flag) {
        // let copies already in flight land before the CTA exits
        int s = stage;
        uint32_t ph = phase;
        for (int i = 0; i < min(issued, kStages); ++i) {
          if (--s < 0) { s = kStages - 1; ph ^= 1u; }
          wait_ns(&full[s], ph, 100000000ull);
          if ((sf_last >> s) & 1u) wait_ns(&sf_full[s], ((sf_phase >> s) & 1u) ^ 1u, 100000000ull);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0, g = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      const uint32_t acc0 = tmem, acc1 = tmem + BN;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        const int tn = t / tiles_m;
        const uint32_t shift = (tn & 1) ? 2u : 0u;   // the tile starts 64 rows into its first B scale chunk
        if (!mbar_wait(acc_empty, acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        uint32_t accumulate = 0;
        for (int it = 0; it < nk; ++it) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          uint8_t* sA0 = smem + stage * S::kStage;
          uint8_t* sA1 = sA0 + S::kA;
          uint8_t* sB = sA1 + S::kA;
          const uint64_t a0 = make_sdesc(smem_u32(sA0), 16, 1024, kSwizzle128B);
          const uint64_t a1 = make_sdesc(smem_u32(sA1), 16, 1024, kSwizzle128B);
          const uint64_t bd = make_sdesc(smem_u32(sB), 16, 1024, kSwizzle128B);
          if (it < p.num_kt) {
            const int slot = g & 1;
            // the scale warp has copied this K step's scales into the slot
            if (!mbar_wait(&sf_ready[slot], static_cast<uint32_t>(g >> 1) & 1u, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sf = tmem + kSfBase + slot * kSlotCols;
            const uint32_t sfa0 = sf, sfa1 = sf + 16, sfb = sf + 32;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint64_t koff = static_cast<uint64_t>((j * 32) >> 4);
              if (nv) {
                const uint32_t id = idesc_fp4(128, BN, false, 0, 0);
                mma_nvf4(acc0, a0 + koff, bd + koff, id, sfa0 + 4 * j, sfb + 8 * j + shift, accumulate);
                mma_nvf4(acc1, a1 + koff, bd + koff, id, sfa1 + 4 * j, sfb + 8 * j + shift, accumulate);
              } else {
                const uint32_t sid = 2u * (j & 1);
                const uint32_t id = idesc_fp4(128, BN, true, sid, sid);
                const uint32_t sb = (sfb + 8 * (j >> 1) + shift) | (sid << 30);
                mma_mxf4(acc0, a0 + koff, bd + koff, id, (sfa0 + 4 * (j >> 1)) | (sid << 30), sb, accumulate);
                mma_mxf4(acc1, a1 + koff, bd + koff, id, (sfa1 + 4 * (j >> 1)) | (sid << 30), sb, accumulate);
              }
              accumulate = 1;
            }
            tc_commit(&sf_free[slot]);
            ++g;
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint64_t koff = static_cast<uint64_t>((j * 32) >> 4);
              const uint32_t id = idesc_bf16(128, BN, false, false);
              mma_bf16(acc0, a0 + koff, bd + koff, id, accumulate);
              mma_bf16(acc1, a1 + koff, bd + koff, id, accumulate);
              accumulate = 1;
            }
          }
          tc_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(acc_full);
        acc_phase ^= 1u;
      }
      if (*abort_flag) {
        // wait for MMAs already issued before the TMEM is freed
        tc_commit(acc_full);
        wait_ns(acc_full, acc_phase, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp == kSfWarp) {
    // ------------------------------------------------------------ scale copies
    // K step g's scales go into slot g & 1 once the MMAs of step g - 2 (the
    // slot's last readers) have retired and the step's scale chunks are in
    // shared memory (sf_full, counted in FP4 steps only), committed to
    // sf_ready[slot]; the copies of step g + 1 run while the MMAs of step g
    // are issued.
    if (lane == 0) {
      int stage = 0, g = 0;
      uint32_t sf_phase = 0;   // bit s: parity of sf_full[s]'s next phase
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        for (int it = 0; it < nk; ++it) {
          if (it < p.num_kt) {
            const int slot = g & 1;
            if (g >= 2) {
              if (!mbar_wait(&sf_free[slot], static_cast<uint32_t>((g >> 1) - 1) & 1u, abort_flag)) { ok = false; break; }
            }
            if (!mbar_wait(&sf_full[stage], (sf_phase >> stage) & 1u, abort_flag)) { ok = false; break; }
            sf_phase ^= 1u << stage;
            tc_fence_after();
            uint8_t* sSFA0 = smem + stage * S::kStage + 2 * S::kA + S::kB;
            uint8_t* sSFA1 = sSFA0 + S::kSFA;
            uint8_t* sSFB = sSFA1 + S::kSFA;
            const uint32_t sf = tmem + kSfBase + slot * kSlotCols;
            const uint32_t sfa0 = sf, sfa1 = sf + 16, sfb = sf + 32;
            for (int a = 0; a < atoms_per_kt; ++a) {
              tc_cp_32x128b_warpx4(sfa0 + 4 * a, make_sdesc(smem_u32(sSFA0 + 512 * a), 0, 128, kSwizzleNone));
              tc_cp_32x128b_warpx4(sfa1 + 4 * a, make_sdesc(smem_u32(sSFA1 + 512 * a), 0, 128, kSwizzleNone));
              for (int h = 0; h < 2; ++h)
                tc_cp_32x128b_warpx4(sfb + 8 * a + 4 * h,
                                     make_sdesc(smem_u32(sSFB + 2048 * h + 512 * a), 0, 128, kSwizzleNone));
            }
            tc_commit(&sf_ready[slot]);
            ++g;
          }
          if (++stage == kStages) stage = 0;
        }
      }
      // copies still in flight land before the TMEM is freed
      if (g >= 1) wait_ns(&sf_ready[(g - 1) & 1], static_cast<uint32_t>((g - 1) >> 1) & 1u, 100000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;               // TMEM lane quadrant of this warp
    const int h = (warp - 2) >> 2;        // M half (accumulator)
    float alpha = 1.f;
    if (p.ts_a) alpha = __fmul_rn(alpha, *p.ts_a);
    if (p.ts_b) alpha = __fmul_rn(alpha, *p.ts_b);
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      const int tm = t % tiles_m, tn = t / tiles_m;
      if (!mbar_wait(acc_full, acc_phase, abort_flag)) break;
      tc_fence_after();
      acc_phase ^= 1u;
      const int64_t row = static_cast<int64_t>(tm) * 256 + 128 * h + 32 * q + lane;
      const bool row_ok = row < p.M;
      const uint32_t tbase = tmem + (static_cast<uint32_t>(32 * q) << 16) + h * BN;
      const int64_t col0 = static_cast<int64_t>(tn) * BN;
      if (p.c_dtype != METIS_F32 && col0 + BN <= p.N && p.vec16_ok) {
        // bf16, full-width tile: the whole row fits in registers as packed
        // pairs, so the accumulator is released before any store
        uint32_t pk[BN / 2];
#pragma unroll
        for (int cc = 0; cc < BN / 16; ++cc) {
          uint32_t v[16];
          tmem_ld16(tbase + 16 * cc, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const __nv_bfloat16 lo = __float2bfloat16_rn(__fmul_rn(alpha, __uint_as_float(v[2 * e])));
            const __nv_bfloat16 hi = __float2bfloat16_rn(__fmul_rn(alpha, __uint_as_float(v[2 * e + 1])));
            pk[8 * cc + e] = static_cast<uint32_t>(__bfloat16_as_ushort(lo)) |
                             (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
        if (!row_ok) continue;
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.C) + row * p.ldc + col0);
#pragma unroll
        for (int c = 0; c < BN / 8; ++c) dst[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        continue;
      }
      // otherwise drained 32 columns at a time and released after the last load
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t v[32];
        tmem_ld16(tbase + 32 * cc, v);
        tmem_ld16(tbase + 32 * cc + 16, v + 16);
        tmem_ld_wait();
        if (cc == BN / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(acc_empty);
        }
        if (!row_ok) continue;
        const int64_t cb = col0 + 32 * cc;
        if (p.c_dtype == METIS_F32) {
          float* dst = reinterpret_cast<float*>(p.C) + row * p.ldc;
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            const int64_t col = cb + c;
            const float4 f = make_float4(__fmul_rn(alpha, __uint_as_float(v[c])), __fmul_rn(alpha, __uint_as_float(v[c + 1])),
                                         __fmul_rn(alpha, __uint_as_float(v[c + 2])), __fmul_rn(alpha, __uint_as_float(v[c + 3])));
            if (col + 3 < p.N && p.vec_ok) {
              *reinterpret_cast<float4*>(dst + col) = f;
            } else {
              const float fe[4] = {f.x, f.y, f.z, f.w};
              for (int e = 0; e < 4; ++e)
                if (col + e < p.N) dst[col + e] = fe[e];
            }
          }
        } else {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.C) + row * p.ldc;
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            const int64_t col = cb + c;
            __nv_bfloat16 b[4];
            for (int e = 0; e < 4; ++e) b[e] = __float2bfloat16_rn(__fmul_rn(alpha, __uint_as_float(v[c + e])));
            if (col + 3 < p.N && p.vec_ok) {
              uint2 u;
              u.x = static_cast<uint32_t>(__bfloat16_as_ushort(b[0])) | (static_cast<uint32_t>(__bfloat16_as_ushort(b[1])) << 16);
              u.y = static_cast<uint32_t>(__bfloat16_as_ushort(b[2])) | (static_cast<uint32_t>(__bfloat16_as_ushort(b[3])) << 16);
              *reinterpret_cast<uint2*>(dst + col) = u;
            } else {
              for (int e = 0; e < 4; ++e)
                if (col + e < p.N) dst[col + e] = b[e];
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && *abort_flag) report(p.dev_status, METIS_DEV_TIMEOUT);
}

// Deterministic split-K reduction: C = alpha * sum_s partial[s] (+ nothing).
__global__ void splitk_reduce_kernel(const float* partial, int splits, int64_t M, int64_t N, const float* ts_a,
                                     const float* ts_b, void* C, int c_dtype, int64_t ldc) {
  const int64_t total = M * N;
  float alpha = 1.f;
  if (ts_a) alpha = __fmul_rn(alpha, *ts_a);
  if (ts_b) alpha = __fmul_rn(alpha, *ts_b);
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float s = 0.f;
    for (int k = 0; k < splits; ++k) s += partial[k * total + i];
    const int64_t r = i / N, c = i - r * N;
    const float v = __fmul_rn(alpha, s);
    if (c_dtype == METIS_F32)
      reinterpret_cast<float*>(C)[r * ldc + c] = v;
    else
      reinterpret_cast<__nv_bfloat16*>(C)[r * ldc + c] = __float2bfloat16_rn(v);
  }
}

}  // namespace

int gemm_effective_splits(int64_t K, int splits) {
  const int num_kt = static_cast<int>((K + 255) / 256);
  int s = splits < 1 ? 1 : splits;
  if (s > num_kt) s = num_kt;
  // every split must own at least one K tile (an empty split would leave
  // its accumulator unwritten): the fewest splits of the same length
  const int per = (num_kt + s - 1) / s;
  return (num_kt + per - 1) / per;
}

namespace {

template <int BN, int STAGES, int CTAS>
cudaError_t launch_bn(const GemmParams& p, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& la,
                      const CUtensorMap& lb, int tiles, cudaStream_t s) {
  const int bytes = Smem<BN, STAGES>::kBytes;
  if (!ensure_smem(reinterpret_cast<const void*>(gemm_fp4_kernel<BN, STAGES, CTAS>), bytes))
    return cudaErrorInvalidValue;
  const int slots = device_sm_count() * CTAS;
  const int grid = tiles < slots ? tiles : slots;
  gemm_fp4_kernel<BN, STAGES, CTAS><<<grid, kThreads, bytes, s>>>(p, a, b, la, lb);
  return cudaGetLastError();
}

cudaError_t launch_wide(const GemmParams& p, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& la,
                        const CUtensorMap& lb, int tiles, cudaStream_t s) {
  const int bytes = WideSmem::kBytes;
  if (!ensure_smem(reinterpret_cast<const void*>(gemm_fp4_wide_kernel), bytes)) return cudaErrorInvalidValue;
  const int slots = device_sm_count();
  const int grid = tiles < slots ? tiles : slots;
  gemm_fp4_wide_kernel<<<grid, kThreads, bytes, s>>>(p, a, b, la, lb);
  return cudaGetLastError();
}

CUresult fp4_map(CUtensorMap* m, const uint8_t* codes, int64_t rows, int64_t inner, uint32_t box_rows) {
  const uint64_t dims[2] = {static_cast<uint64_t>(inner / 2), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(inner / 2)};
  const uint32_t box[2] = {128, box_rows};
  return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, codes, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B);
}

CUresult bf16_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, uint32_t box_rows) {
  const uint64_t dims[2] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(cols) * 2};
  const uint32_t box[2] = {64, box_rows};
  return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

metis_status run_gemm_fp4(const GemmCall& g, cudaStream_t s) {
  GemmParams p{};
  p.fmt = g.fmt;
  p.M = static_cast<int>(g.M);
  p.N = static_cast<int>(g.N);
  p.num_kt = static_cast<int>((g.K + 255) / 256);
  const int64_t sc_cols = tc_scale_cols(g.fmt, g.K);
  p.sfa = g.a_scales;
  p.sfb = g.b_scales;
  p.sfa_chunks = sc_cols / 4;
  p.sfb_chunks = sc_cols / 4;
  p.sfb_rows = tc_scale_rows(g.N);
  p.ts_a = g.fmt == METIS_NVFP4 ? g.a_tensor_scale : nullptr;
  p.ts_b = g.fmt == METIS_NVFP4 ? g.b_tensor_scale : nullptr;
  p.lr_chunks = g.lr_k / 64;
  p.C = g.C;
  p.c_dtype = g.c_dtype;
  p.ldc = g.ldc;
  p.vec_ok = (g.ldc % 4 == 0) && ((reinterpret_cast<uintptr_t>(g.C) & 15u) == 0);
  p.vec16_ok = (g.ldc % 8 == 0) && ((reinterpret_cast<uintptr_t>(g.C) & 15u) == 0);
  p.dev_status = g.dev_status;
  p.splits = gemm_effective_splits(g.K, g.splits);
  p.partial = g.partial;
  if (p.splits > 1 && !p.partial) return METIS_ERR_ARG;
  if (p.splits > 1 && p.lr_chunks) return METIS_ERR_ARG;
  // The wide tile (two 128-row halves sharing a 192-row B tile) covers 1.5
  // times the work of a 128 x 256 tile and, measured on an NVFP4
  // 8192 x 4096 x 4096 product, runs a unit of work 4.5 % faster
  // (17.4 against 18.2 us per 128 x 256 x 4096 unit).  It is taken for
  // unsplit products when its rounds of tiles over the SMs cost less.
  bool wide = false;
  if (g.bn == 256 && p.splits == 1 && g.M >= 256 && g.N >= 384) {
    const int64_t sms = device_sm_count();
    const int64_t rounds_n = (((g.M + 127) / 128) * ((g.N + 255) / 256) + sms - 1) / sms;
    const int64_t rounds_w = (((g.M + 255) / 256) * ((g.N + kWideBN - 1) / kWideBN) + sms - 1) / sms;
    wide = rounds_w * 1433 < rounds_n * 1000;   // 1.5 x 0.955
  }
  const int bn = wide ? kWideBN : g.bn;
  CUtensorMap ma, mb, mla, mlb;
  if (fp4_map(&ma, g.a_codes, g.M, g.K, 128) != CUDA_SUCCESS) return fail(METIS_ERR_CUDA, "gemm_fp4 tensor map");
  if (fp4_map(&mb, g.b_codes, g.N, g.K, static_cast<uint32_t>(bn)) != CUDA_SUCCESS) return fail(METIS_ERR_CUDA, "gemm_fp4 tensor map");
  if (p.lr_chunks) {
    if (bf16_map(&mla, g.lr_a, g.M, g.lr_k, 128) != CUDA_SUCCESS) return fail(METIS_ERR_CUDA, "gemm_fp4 tensor map");
    if (bf16_map(&mlb, g.lr_b, g.N, g.lr_k, static_cast<uint32_t>(bn)) != CUDA_SUCCESS) return fail(METIS_ERR_CUDA, "gemm_fp4 tensor map");
  } else {
    mla = ma;
    mlb = mb;
  }
  const int tiles = static_cast<int>(((g.M + 127) / 128) * ((g.N + bn - 1) / bn)) * p.splits;
  cudaError_t e;
  if (wide)
    e = launch_wide(p, ma, mb, mla, mlb, static_cast<int>(((g.M + 255) / 256) * ((g.N + bn - 1) / bn)), s);
  else if (bn == 256)
    e = launch_bn<256, 4, 1>(p, ma, mb, mla, mlb, tiles, s);
  else if (bn == 128)
    e = launch_bn<128, 4, 1>(p, ma, mb, mla, mlb, tiles, s);
  else if (bn == 64)
    e = launch_bn<64, 4, 1>(p, ma, mb, mla, mlb, tiles, s);
  else
    return METIS_ERR_ARG;
  if (e != cudaSuccess) return fail(METIS_ERR_CUDA, "gemm_fp4 launch", cudaGetErrorString(e));
  if (p.splits > 1 && g.C) {
    const int64_t total = g.M * g.N;
    int blocks = static_cast<int>((total + 255) / 256);
    if (blocks > device_sm_count() * 8) blocks = device_sm_count() * 8;
    splitk_reduce_kernel<<<blocks, 256, 0, s>>>(p.partial, p.splits, g.M, g.N, p.ts_a, p.ts_b, g.C, g.c_dtype, g.ldc);
  }
  return launch_status();
}

}  // namespace metis
