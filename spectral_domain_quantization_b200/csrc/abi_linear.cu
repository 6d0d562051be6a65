// C ABI: metis_linear_fwd and metis_linear_bwd (see include/metis.h).
//
// Both are built from one operation, the product of two split operands:
//   C = A B,  A = R_A + F_A S_A P_A^T (M x K),  B = R_B + P_B S_B F_B^T (K x N)
//     = R_A R_B + T1 F_B^T + F_A T2
// Source: "Metis: Training LLMs with FP4 Quantization" abstract (W4A4G4
// forward and backward products); SII release section 2.4 item 1; Averis
// paragraphs of the arXiv 2603.10444 retelling (rank-1 mean terms).
//
// Enqueued work for one product:
//   1. T1raw = R_A P_B    FP4 GEMM (N = kB, split-K), or R_A's inner sums when
//                         P_B is the all-ones vector
//   2. T2raw = P_A^T R_B  FP4 GEMM (M = kA, split-K), or R_B's inner sums
//   3. Cab  = P_A^T P_B   small dot-product kernel (both operands split)
//   4. LA / LB            bf16 low-rank operands (lowrank.cu)
//   5. C                  FP4 GEMM over K plus the low-rank chunks, one launch
#include "abi_common.h"
#include "common.cuh"
#include "gemm_fp4.h"
#include "lowrank.h"

namespace metis {

namespace {

metis_status check_operand(const metis_operand* op, int64_t free_dim, int64_t K, int fmt) {
  if (!op || !op->R) return METIS_ERR_NULL;
  METIS_TRY(check_fp4(op->R, free_dim, K, fmt));
  if (op->k < 0 || op->k > 128) return METIS_ERR_ARG;
  if (op->flags & ~METIS_REQUANT_LOWRANK) return METIS_ERR_ARG;
  if (op->k == 0) return METIS_OK;
  if (op->P) {
    METIS_TRY(check_fp4(op->P, op->k, K, fmt));
  } else if (op->k != 1) {
    return METIS_ERR_ARG;
  }
  if (op->F) {
    METIS_TRY(check_fp4(op->F, op->k, free_dim, fmt));
  } else if (op->k != 1) {
    return METIS_ERR_ARG;
  }
  return METIS_OK;
}

FactorView view_of(const metis_fp4_tensor* t) {
  FactorView f{};
  if (!t) {
    f.ones = 1;
    return f;
  }
  f.ones = 0;
  f.fmt = t->fmt;
  f.inner = t->inner;
  f.scale_cols = tc_scale_cols(t->fmt, t->inner);
  f.codes = t->codes;
  f.scales = t->scales;
  f.tensor_scale = t->fmt == METIS_NVFP4 ? t->tensor_scale : nullptr;
  return f;
}

int num_kt(int64_t K) { return static_cast<int>((K + 255) / 256); }

int pick_splits(int64_t tiles, int64_t K) {
  const int64_t sms = device_sm_count();
  int64_t s = tiles >= sms ? 1 : sms / tiles;
  if (s > num_kt(K)) s = num_kt(K);
  if (s > 16) s = 16;
  return static_cast<int>(s < 1 ? 1 : s);
}

GemmCall base_call(const metis_fp4_tensor* a, const metis_fp4_tensor* b, int64_t M, int64_t N, int64_t K,
                   int32_t* dev_status) {
  GemmCall g{};
  g.fmt = a->fmt;
  g.M = M;
  g.N = N;
  g.K = K;
  g.a_codes = a->codes;
  g.a_scales = a->scales;
  g.a_tensor_scale = a->tensor_scale;
  g.b_codes = b->codes;
  g.b_scales = b->scales;
  g.b_tensor_scale = b->tensor_scale;
  g.dev_status = dev_status;
  g.splits = 1;
  return g;
}

int bn_for(int64_t N) { return N >= 256 ? 256 : (N > 64 ? 128 : 64); }

struct ProductPlan {
  int ka, kb;
  int64_t lr_k;
  int s1, s2;
};

ProductPlan plan(const metis_operand* A, const metis_operand* B, int64_t M, int64_t N, int64_t K) {
  ProductPlan p{};
  p.ka = A->k;
  p.kb = B->k;
  const int w = 2 * p.ka + 2 * p.kb;
  p.lr_k = w ? (w + 63) / 64 * 64 : 0;
  p.s1 = (p.kb && B->P) ? pick_splits((M + 127) / 128, K) : 1;
  p.s2 = (p.ka && A->P) ? pick_splits((N + 255) / 256, K) : 1;
  return p;
}

// Workspace of one product; with ws.base == NULL only sizes are summed.
struct ProductBuffers {
  __nv_bfloat16 *la = nullptr, *lb = nullptr;
  float *t1 = nullptr, *t1p = nullptr, *t2 = nullptr, *t2p = nullptr, *cab = nullptr, *cabp = nullptr;
  float* t1full = nullptr;      // re-quantized T1: its float32 values
  unsigned* amax = nullptr;     // [2]: max |T1|, max |T2| (NVFP4)
};

ProductBuffers carve(const ProductPlan& p, const metis_operand* A, const metis_operand* B, int64_t M,
                     int64_t N, int64_t K, Carver& ws) {
  ProductBuffers b;
  if (!p.lr_k) return b;
  b.la = ws.take<__nv_bfloat16>(static_cast<size_t>(M) * p.lr_k);
  b.lb = ws.take<__nv_bfloat16>(static_cast<size_t>(N) * p.lr_k);
  if (p.kb && B->P) {
    b.t1 = ws.take<float>(static_cast<size_t>(M) * p.kb);
    if (p.s1 > 1) b.t1p = ws.take<float>(static_cast<size_t>(p.s1) * M * p.kb);
  }
  if (p.ka && A->P) {
    b.t2 = ws.take<float>(static_cast<size_t>(p.ka) * N);
    if (p.s2 > 1) b.t2p = ws.take<float>(static_cast<size_t>(p.s2) * p.ka * N);
  }
  if (p.ka && p.kb) {
    b.cab = ws.take<float>(static_cast<size_t>(p.ka) * p.kb);
    b.cabp = ws.take<float>(static_cast<size_t>(cab_parts(K, device_sm_count())) * p.ka * p.kb);
  }
  if (p.kb && (B->flags & METIS_REQUANT_LOWRANK)) b.t1full = ws.take<float>(static_cast<size_t>(M) * p.kb);
  if ((p.kb && (B->flags & METIS_REQUANT_LOWRANK)) || (p.ka && (A->flags & METIS_REQUANT_LOWRANK)))
    b.amax = ws.take<unsigned>(2);
  return b;
}

metis_status check_product(const metis_operand* A, const metis_operand* B, int64_t M, int64_t N, int64_t K) {
  if (!A || !B || !A->R || !B->R) return METIS_ERR_NULL;
  if (M <= 0 || N <= 0 || K <= 0 || K % 32) return METIS_ERR_SHAPE;
  // the GEMM indexes rows, columns and K tiles of one product in 32 bits
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return METIS_ERR_SHAPE;
  const int fmt = A->R->fmt;
  if (!valid_fmt(fmt)) return METIS_ERR_ARG;
  METIS_TRY(check_operand(A, M, K, fmt));
  METIS_TRY(check_operand(B, N, K, fmt));
  if (A->k && !A->P && !B->R->inner_sum) return METIS_ERR_NULL;  // ones . R_B needs R_B's sums
  if (B->k && !B->P && !A->R->inner_sum) return METIS_ERR_NULL;
  return METIS_OK;
}

metis_status enqueue_product(const metis_operand* A, const metis_operand* B, int64_t M, int64_t N, int64_t K,
                             void* C, int c_dtype, int64_t ldc, Carver& ws, int32_t* dev_status,
                             cudaStream_t s) {
  const ProductPlan p = plan(A, B, M, N, K);
  const ProductBuffers b = carve(p, A, B, M, N, K, ws);
  if (!ws.base) return METIS_OK;
  const int sms = device_sm_count();
  LowRankArgs la{};
  if (p.lr_k) {
    la.M = M;
    la.N = N;
    la.ka = p.ka;
    la.kb = p.kb;
    la.lr_k = p.lr_k;
    la.fa = view_of(p.ka ? A->F : nullptr);
    la.fb = view_of(p.kb ? B->F : nullptr);
    la.s_a = A->S;
    la.s_b = B->S;
    la.ts_ra = A->R->fmt == METIS_NVFP4 ? A->R->tensor_scale : nullptr;
    la.ts_rb = B->R->fmt == METIS_NVFP4 ? B->R->tensor_scale : nullptr;
    la.la = b.la;
    la.lb = b.lb;
    la.fmt = A->R->fmt;
    la.requant_t1 = p.kb && (B->flags & METIS_REQUANT_LOWRANK);
    la.requant_t2 = p.ka && (A->flags & METIS_REQUANT_LOWRANK);
    la.t1full = b.t1full;
    la.amax1 = b.amax;
    la.amax2 = b.amax ? b.amax + 1 : nullptr;
    if (p.kb) {
      if (B->P) {
        GemmCall g = base_call(A->R, B->P, M, p.kb, K, dev_status);
        g.bn = p.kb <= 64 ? 64 : 128;
        g.c_dtype = METIS_F32;
        g.ldc = p.kb;
        g.splits = p.s1;
        g.partial = b.t1p;
        const int splits = gemm_effective_splits(K, p.s1);
        if (splits > 1) {
          // keep the partial sums: build_la adds them (no separate reduction)
          g.C = nullptr;
          la.t1part = b.t1p;
          la.t1_splits = splits;
          la.t1_ts_a = A->R->fmt == METIS_NVFP4 ? A->R->tensor_scale : nullptr;
          la.t1_ts_b = B->P->fmt == METIS_NVFP4 ? B->P->tensor_scale : nullptr;
        } else {
          g.C = b.t1;
          la.t1raw = b.t1;
          la.t1_ld = p.kb;
        }
        METIS_TRY(run_gemm_fp4(g, s));
      } else {
        la.t1raw = A->R->inner_sum;  // R_A 1
        la.t1_ld = 1;
      }
    }
    if (p.ka) {
      if (A->P) {
        GemmCall g = base_call(A->P, B->R, p.ka, N, K, dev_status);
        g.bn = bn_for(N);
        g.C = b.t2;
        g.c_dtype = METIS_F32;
        g.ldc = N;
        g.splits = p.s2;
        g.partial = b.t2p;
        METIS_TRY(run_gemm_fp4(g, s));
        la.t2raw = b.t2;
        la.t2_ld = N;
      } else {
        la.t2raw = B->R->inner_sum;  // 1^T R_B
        la.t2_ld = N;
      }
    }
    if (p.ka && p.kb) {
      // an all-ones P contributes 1 at every position of the contraction
      if (!launch_cab(view_of(A->P), view_of(B->P), K, p.ka, p.kb, b.cabp, b.cab, sms, s))
        return fail(METIS_ERR_CUDA, "low-rank core product shared-memory attribute");
      la.cab = b.cab;
    }
    launch_build_lowrank(la, sms, s);
  }
  GemmCall g = base_call(A->R, B->R, M, N, K, dev_status);
  g.bn = bn_for(N);
  g.lr_a = b.la;
  g.lr_b = b.lb;
  g.lr_k = p.lr_k;
  g.C = C;
  g.c_dtype = c_dtype;
  g.ldc = ldc;
  METIS_TRY(run_gemm_fp4(g, s));
  return launch_status();
}

size_t product_workspace(const metis_operand* A, const metis_operand* B, int64_t M, int64_t N, int64_t K) {
  Carver c(nullptr);
  carve(plan(A, B, M, N, K), A, B, M, N, K, c);
  return c.used;
}

metis_status check_out(void* C, int dt, int64_t ld, int64_t cols) {
  if (!C) return METIS_ERR_NULL;
  if (dt != METIS_F32 && dt != METIS_BF16) return METIS_ERR_ARG;
  if (ld < cols) return METIS_ERR_SHAPE;
  return METIS_OK;
}

}  // namespace

}  // namespace metis

using namespace metis;

extern "C" metis_status metis_linear_fwd(const metis_operand* X, const metis_operand* W, int64_t M, int64_t N,
                                         int64_t K, void* Y, int32_t y_dtype, int64_t ldy, void* workspace,
                                         size_t* workspace_bytes, int32_t* dev_status, void* stream) {
  if (!workspace_bytes) return METIS_ERR_NULL;
  METIS_TRY(check_product(X, W, M, N, K));
  METIS_TRY(check_out(Y, y_dtype, ldy, N));
  const size_t need = product_workspace(X, W, M, N, K);
  if (!workspace) {
    *workspace_bytes = need;
    return METIS_OK;
  }
  if (*workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return METIS_ERR_WORKSPACE;
  if (!device_is_sm100()) return METIS_ERR_UNSUPPORTED;
  Carver ws(workspace);
  return enqueue_product(X, W, M, N, K, Y, y_dtype, ldy, ws, dev_status, static_cast<cudaStream_t>(stream));
}

extern "C" metis_status metis_linear_bwd(const metis_operand* dY_n, const metis_operand* Wt,
                                         const metis_operand* Xt, const metis_operand* dY_m, int64_t M,
                                         int64_t N, int64_t K, void* dX, int64_t ld_dx, void* dW, int64_t ld_dw,
                                         int32_t out_dtype, void* workspace, size_t* workspace_bytes,
                                         int32_t* dev_status, void* stream) {
  if (!workspace_bytes) return METIS_ERR_NULL;
  if (!dX && !dW) return METIS_ERR_NULL;
  // dX (M x K) = dY (M x N) W^T (N x K): contraction N
  if (dX) {
    METIS_TRY(check_product(dY_n, Wt, M, K, N));
    METIS_TRY(check_out(dX, out_dtype, ld_dx, K));
  }
  // dW (K x N) = X^T (K x M) dY (M x N): contraction M
  if (dW) {
    METIS_TRY(check_product(Xt, dY_m, K, N, M));
    METIS_TRY(check_out(dW, out_dtype, ld_dw, N));
  }
  size_t need = 0;
  if (dX) need = product_workspace(dY_n, Wt, M, K, N);
  if (dW) {
    const size_t n2 = product_workspace(Xt, dY_m, K, N, M);
    need = n2 > need ? n2 : need;
  }
  if (!workspace) {
    *workspace_bytes = need;
    return METIS_OK;
  }
  if (*workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return METIS_ERR_WORKSPACE;
  if (!device_is_sm100()) return METIS_ERR_UNSUPPORTED;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dX) {
    Carver ws(workspace);
    METIS_TRY(enqueue_product(dY_n, Wt, M, K, N, dX, out_dtype, ld_dx, ws, dev_status, s));
  }
  if (dW) {
    Carver ws(workspace);  // runs after dX on the same stream: the region is reused
    METIS_TRY(enqueue_product(Xt, dY_m, K, N, M, dW, out_dtype, ld_dw, ws, dev_status, s));
  }
  return METIS_OK;
}
