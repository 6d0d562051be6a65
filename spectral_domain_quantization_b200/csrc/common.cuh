// Device helpers shared by the kernels: status bits, bounded waits, mbarriers,
// TMA / bulk copies, tcgen05 (TMEM allocation, MMA, copies, loads) and the
// shared-memory / instruction descriptors of the sm_100a tensor cores.
//
// Descriptor bit layouts follow the PTX ISA description of tcgen05 matrix and
// instruction descriptors (the same layouts CUTLASS's cute/arch/mma_sm100_desc
// encodes): shared-memory descriptor = start address >> 4 in bits 0-13, leading
// byte offset >> 4 in bits 16-29, stride byte offset >> 4 in bits 32-45,
// version 1 in bits 46-47, swizzle mode in bits 61-63.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/metis.h"

#define MDEV __device__ __forceinline__

namespace metis {

// ---------------------------------------------------------------------------
// status and bounded waits
// ---------------------------------------------------------------------------

// A wait that has not finished after this many nanoseconds gives up, sets
// METIS_DEV_TIMEOUT and lets the kernel wind down.
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;

MDEV uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

MDEV void report(int32_t* dev_status, int32_t bits) {
  if (dev_status) atomicOr(dev_status, bits);
}

__host__ __device__ inline int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ inline int64_t imax64(int64_t a, int64_t b) { return a > b ? a : b; }

MDEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------

MDEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

MDEV void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

MDEV void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

MDEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

MDEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

MDEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar`.  Returns false once *abort is set (by this
// or another thread) or after limit_ns; a timeout sets *abort.
MDEV bool mbar_wait_for(uint64_t* bar, uint32_t parity, volatile int* abort, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        *abort = 1;
        return false;
      }
    }
  }
}

// The wait every kernel uses: limit kWaitTimeoutNs.
MDEV bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return mbar_wait_for(bar, parity, abort, kWaitTimeoutNs);
}

// ---------------------------------------------------------------------------
// thread-block clusters (distributed shared memory)
// ---------------------------------------------------------------------------

MDEV uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
MDEV uint32_t map_to_rank(uint32_t smem_addr, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_addr), "r"(rank));
  return out;
}

// Every thread of every CTA of the cluster arrives; the waits see the other
// CTAs' shared-memory writes made before their arrival.
MDEV void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

MDEV float4 ld_cluster_f32x4(uint32_t cluster_addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(cluster_addr)
               : "memory");
  return v;
}

MDEV double2 ld_cluster_f64x2(uint32_t cluster_addr) {
  double2 v;
  asm volatile("ld.shared::cluster.v2.f64 {%0, %1}, [%2];" : "=d"(v.x), "=d"(v.y) : "r"(cluster_addr) : "memory");
  return v;
}

// ---------------------------------------------------------------------------
// TMA and bulk copies (global -> shared, completion on an mbarrier)
// ---------------------------------------------------------------------------

MDEV void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// bytes: multiple of 16; both addresses 16-byte aligned.
MDEV void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

MDEV void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory, MMA, copies, loads
// ---------------------------------------------------------------------------

// Warp-wide.  Writes the allocated TMEM base address to *dst (shared memory).
MDEV void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
}

MDEV void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

MDEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

MDEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
MDEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrive on `bar` once all previously issued tcgen05 ops of this thread finish.
MDEV void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// D (+)= A * B, bf16 inputs, fp32 accumulator in TMEM.
MDEV void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                   uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Block-scaled FP4 MMA, NVFP4: E2M1 x E2M1 with one UE4M3 scale per 16 along K.
MDEV void mma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                   uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], "
      "[%6], p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Block-scaled FP4 MMA, MXFP4: E2M1 x E2M1 with one UE8M0 scale per 32 along K.
MDEV void mma_mxf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                   uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], "
      "p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Shared memory -> TMEM copy of 32 rows x 128 bits, replicated to the four
// 32-lane groups (used for block-scale factors).
MDEV void tc_cp_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

MDEV void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 bits, 16 consecutive columns per thread.
MDEV void tmem_ld16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// ---------------------------------------------------------------------------
// descriptors
// ---------------------------------------------------------------------------

enum : uint32_t { kSwizzleNone = 0, kSwizzle128B = 2 };

// Shared-memory matrix descriptor.
MDEV uint64_t make_sdesc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                         uint32_t swizzle) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(swizzle & 7u) << 61;
  return d;
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major,
                                                  bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn_major) << 15) |
         (static_cast<uint32_t>(b_mn_major) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor, block-scaled FP4 (E2M1 x E2M1), K-major A and B.
// ue8m0: scale type (1 = E8M0 for MXFP4, 0 = E4M3 for NVFP4); sf ids select
// the byte of the 32-bit TMEM scale column a K=64 step starts at.
__host__ __device__ constexpr uint32_t idesc_fp4(int M, int N, bool ue8m0, uint32_t a_sf_id,
                                                 uint32_t b_sf_id) {
  return (b_sf_id << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(ue8m0) << 23) | (static_cast<uint32_t>(M >> 4) << 24) |
         (a_sf_id << 29);
}

// ---------------------------------------------------------------------------
// FP4 codecs (bit-exact with the float32 rules documented in metis.h)
// ---------------------------------------------------------------------------

// E2M1 code of a scaled float32: nearest of {0,.5,1,1.5,2,3,4,6}, ties to the
// even code, saturating at 6, sign bit from the float's sign bit.
MDEV uint32_t e2m1_code(float q) {
  const float a = fabsf(q);
  uint32_t c = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) +
               (a >= 3.5f) + (a > 5.0f);
  return c | ((__float_as_uint(q) >> 28) & 8u);
}

// E2M1 codes of 8 values packed into 32 bits (element i in bits 4i..4i+3),
// by the hardware conversion: round to nearest even, saturating at 6, sign
// kept on zero -- the same rule as e2m1_code.  The instruction converts a
// pair with its first operand in the upper nibble.
MDEV uint32_t e2m1_pack8(const float* q) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(q[0]), "f"(q[1]), "f"(q[2]), "f"(q[3]), "f"(q[4]), "f"(q[5]), "f"(q[6]), "f"(q[7]));
  return r;
}

// Value of an E2M1 code.  Twice the magnitudes {0,1,2,3,4,6,8,12} are packed
// as nibbles of one constant, so the lookup stays in registers.
__host__ __device__ inline float e2m1_value(uint32_t code) {
  const float v = static_cast<float>((0xC8643210u >> (4u * (code & 7u))) & 15u) * 0.5f;
  return (code & 8u) ? -v : v;
}

// E4M3 code of t >= 0 by the hardware conversion (round to nearest even,
// saturating finite values and infinity at 448 = 0x7E): the same code as
// e4m3_code_ref below for every t >= 0.
MDEV uint32_t e4m3_code(float t) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(0.f), "f"(t));
  return d & 0xFFu;
}

// E4M3 code of t >= 0: round to nearest even, saturating at 448 (0x7E),
// written out from the format's definition.
MDEV uint32_t e4m3_code_ref(float t) {
  if (!(t > 0.f)) return 0u;
  if (t >= 464.f) return 0x7Eu;  // half-way to the non-finite 480 and above
  const uint32_t bits = __float_as_uint(t);
  const int e = static_cast<int>(bits >> 23) - 127;
  if (e < -10) return 0u;  // below half the smallest subnormal 2^-9
  if (e < -6) {            // subnormal range, quantum 2^-9
    return static_cast<uint32_t>(rintf(__fmul_rn(t, 512.f)));
  }
  const float scale = __uint_as_float(static_cast<uint32_t>(127 + 3 - e) << 23);
  uint32_t m = static_cast<uint32_t>(rintf(__fmul_rn(t, scale)));  // 8..16
  int E = e;
  if (m == 16u) {
    m = 8u;
    E += 1;
  }
  uint32_t code = (static_cast<uint32_t>(E + 7) << 3) | (m - 8u);
  return code > 0x7Eu ? 0x7Eu : code;
}

__host__ __device__ inline float e4m3_value(uint32_t code) {
  const uint32_t e = (code >> 3) & 15u, m = code & 7u;
  if (e == 0) return static_cast<float>(m) * 0.001953125f;  // m * 2^-9
  // (8 + m) * 2^(e - 10)
  float p = 1.f;
  int ex = static_cast<int>(e) - 10;
  if (ex >= 0) {
    for (int i = 0; i < ex; ++i) p *= 2.f;
  } else {
    for (int i = 0; i < -ex; ++i) p *= 0.5f;
  }
  return static_cast<float>(8u + m) * p;
}

// floor(log2 a) for finite a > 0 (normal or subnormal).
MDEV int floor_log2(float a) {
  const uint32_t bits = __float_as_uint(a);
  const int ef = static_cast<int>(bits >> 23);
  if (ef > 0) return ef - 127;
  return (31 - __clz(bits & 0x7FFFFFu)) - 149;
}

// 2^k as a float for k in [-126, 127].
MDEV float pow2f(int k) { return __uint_as_float(static_cast<uint32_t>(127 + k) << 23); }

// Byte offset of scale (r, c) in the tensor-core scale layout with C padded
// scale columns.
__host__ __device__ inline int64_t tc_scale_offset(int64_t r, int64_t c, int64_t C) {
  return ((r >> 7) * (C >> 2) + (c >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (c & 3);
}

__host__ __device__ inline int64_t tc_scale_cols(int fmt, int64_t inner) {
  const int64_t bs = fmt == METIS_MXFP4 ? 32 : 16;
  const int64_t per_tile = 256 / bs;
  return ((inner / bs + per_tile - 1) / per_tile) * per_tile;
}

__host__ __device__ inline int64_t tc_scale_rows(int64_t outer) { return (outer + 127) / 128 * 128; }

MDEV float load_elem(const void* X, int dtype, int64_t idx) {
  if (dtype == METIS_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(X)[idx]);
  return reinterpret_cast<const float*>(X)[idx];
}

}  // namespace metis
