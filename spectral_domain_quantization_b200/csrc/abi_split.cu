// C ABI: metis_split (see include/metis.h).
//
// Source: SII release on Metis, section 2.4 item 1 (spectral split into a
// dominant and a long-tail part, randomized dimension reduction); "Metis:
// Training LLMs with FP4 Quantization" abstract and technical framework
// (random projection; sparse random sampling).
//
// Enqueued pipeline (all on `stream`, no host synchronisation):
//   [sample rows -> gather A_s]                      sketch.cu
//   Omega^T (Philox Gaussian / sparse sign, bf16)    sketch.cu
//   Y = A Omega                                      skinny_gemm.cu (tcgen05;
//                                                    each pass also writes the
//                                                    operand of the next one
//                                                    and its Gram partials)
//   q = 0: Q = orth(Y), two CholeskyQR passes        small_linalg.cu
//   q >= 1: Y as is, then q x { Q1 = orth(A^T Y); Y = A Q1; Q = orth(Y) },
//           one CholeskyQR pass each
//   Z = B^T = A^T Q, C = Z^T Z                       skinny pass + Gram
//   C = W diag(sigma^2) W^T, top k                   core_eig.cu (tridiagonal
//                                                    reduction, multisection,
//                                                    twisted factorisation)
//   U = Q W_k, V = Z W_k / sigma, S = sigma          row-block products
//   signs; U_q, V_q                                  quantize.cu
//   R = A - U S V^T, FP4 along n and/or m            residual_quant.cu
// Sampled variant: the steps above on the sampled rows give V_s (n x k);
// then P = A V_s, P^T P = W diag(sigma^2) W^T (this is R_P^T R_P for the QR
// factor of P, so W, sigma are the SVD of R_P), U = P W / sigma, V = V_s W.
#include "abi_common.h"
#include "abi_internal.h"
#include "common.cuh"
#include "kernels.h"
#include "lowrank.h"
#include "residual_quant.h"
#include "sketch.h"
#include "skinny_gemm.h"
#include "small_linalg.h"

namespace metis {

namespace {

static_assert(sizeof(metis_split_params) == 56, "metis_split_params layout (the Python binding mirrors it)");

int round_up(int x, int m) { return (x + m - 1) / m * m; }
int64_t round_up64(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

struct SplitPlan {
  int64_t m, n;          // matrix the range finder runs on (A or A_s) is ms x n
  int64_t ms;            // rows of the range-finder matrix (m or sample_rows)
  int l, lp, k, kp, kq;  // kq = k padded to 16 (sampled P width); kp = k padded to 64
  int64_t ld_m, ld_n;    // padded lengths (multiples of 8) of transposed operands
  int cs_m, cs_n;        // K slices (cluster size) of the A X (rows ms) and A^T X passes
  int cs_m2;             // the A X passes with a two-part (hi / lo) X
  int sampled, fp32;
};

struct SplitBuffers {
  __nv_bfloat16* omt = nullptr;      // [lp][ld_n]
  __nv_bfloat16* a_hi = nullptr;     // fp32 input: bf16 parts (ms x lda)
  __nv_bfloat16* a_lo = nullptr;
  __nv_bfloat16* af_hi = nullptr;    // fp32 input, sampled: parts of the full A
  __nv_bfloat16* af_lo = nullptr;
  void* a_s = nullptr;               // gathered rows (sampled)
  int32_t* idx = nullptr;
  SelectState* sel = nullptr;
  unsigned* hist = nullptr;
  float* Y = nullptr;                // max(m, n) x lp
  float* Q1 = nullptr;               // max(m, n) x lp
  float* Qm = nullptr;               // ms x lp   (range basis)
  float* Zn = nullptr;               // n x lp    (A^T Q)
  __nv_bfloat16* qt = nullptr;       // [2 lp][max(ld_m, ld_n)]
  double* gpart = nullptr;
  double* G = nullptr;
  double* eig_ws = nullptr;          // core eigensolver scratch
  float* Lt = nullptr;     // the Cholesky factor, column by column (launch_cholesky)
  double* eval = nullptr;
  float* evec = nullptr;
  float* Mu = nullptr;
  float* Mv = nullptr;
  float* Vs = nullptr;               // sampled: n x kq
  float* P = nullptr;                // sampled: m x kq
  double* eval2 = nullptr;
  float* evec2 = nullptr;
  float* bmax = nullptr;
  int64_t* bidx = nullptr;
  float* sign = nullptr;
  __nv_bfloat16 *u_hi = nullptr, *u_lo = nullptr, *w_hi = nullptr, *w_lo = nullptr;
  unsigned* amax = nullptr;
};

SplitPlan make_plan(int64_t m, int64_t n, int dtype, const metis_split_params* prm) {
  SplitPlan p{};
  p.m = m;
  p.n = n;
  p.sampled = prm->sample_rows > 0;
  p.ms = p.sampled ? prm->sample_rows : m;
  p.k = prm->k;
  p.l = prm->k + prm->p;
  p.lp = round_up(p.l, 16);
  p.kq = round_up(p.k, 16);
  p.kp = round_up(p.k, 64);
  p.ld_m = round_up64(m, 8);
  p.ld_n = round_up64(n, 8);
  p.fp32 = dtype == METIS_F32;
  const int sms = device_sm_count();
  // passes whose X has two parts (hi / lo; every pass but the sketch's) run
  // fastest with at most 4 K slices per tile (measured: 12.8 against 13.9 us
  // on 4096 x 4096 at 8 slices)
  p.cs_m = skinny_cluster(p.ms, n, sms);
  p.cs_m2 = p.cs_m > 4 ? 4 : p.cs_m;
  p.cs_n = skinny_cluster(n, p.ms, sms);
  if (p.cs_n > 4) p.cs_n = 4;
  return p;
}

SplitBuffers carve(const SplitPlan& p, int64_t lda, Carver& ws) {
  SplitBuffers b;
  const int64_t big = p.m > p.n ? p.m : p.n;
  const int64_t bigld = p.ld_m > p.ld_n ? p.ld_m : p.ld_n;
  b.omt = ws.take<__nv_bfloat16>(static_cast<size_t>(p.lp) * p.ld_n);
  if (p.sampled) {
    b.idx = ws.take<int32_t>(p.ms);
    b.sel = ws.take<SelectState>(1);
    b.hist = ws.take<unsigned>(65536);
    b.a_s = ws.take<uint8_t>(static_cast<size_t>(p.ms) * lda * (p.fp32 ? 4 : 2));
  }
  if (p.fp32) {
    b.a_hi = ws.take<__nv_bfloat16>(static_cast<size_t>(p.ms) * lda);
    b.a_lo = ws.take<__nv_bfloat16>(static_cast<size_t>(p.ms) * lda);
    if (p.sampled) {
      b.af_hi = ws.take<__nv_bfloat16>(static_cast<size_t>(p.m) * lda);
      b.af_lo = ws.take<__nv_bfloat16>(static_cast<size_t>(p.m) * lda);
    }
  }
  const int wmax = p.lp > p.kq ? p.lp : p.kq;
  b.Y = ws.take<float>(static_cast<size_t>(big) * wmax);
  b.Q1 = ws.take<float>(static_cast<size_t>(big) * p.lp);
  b.Qm = ws.take<float>(static_cast<size_t>(p.ms) * p.lp);
  b.Zn = ws.take<float>(static_cast<size_t>(p.n) * p.lp);
  b.qt = ws.take<__nv_bfloat16>(static_cast<size_t>(2 * wmax) * bigld);
  const int64_t gblocks = imax64(gram_blocks(big), apply_blocks(big));  // Gram partials per row block
  b.gpart = ws.take<double>(static_cast<size_t>(gblocks) * wmax * wmax);
  b.G = ws.take<double>(static_cast<size_t>(wmax) * wmax);
  b.eig_ws = reinterpret_cast<double*>(ws.take<uint8_t>(core_eig_workspace(wmax)));
  b.Lt = ws.take<float>(static_cast<size_t>(p.lp) * p.lp);
  b.eval = ws.take<double>(p.lp);
  b.evec = ws.take<float>(static_cast<size_t>(p.lp) * p.lp);
  b.Mu = ws.take<float>(static_cast<size_t>(p.lp) * p.k);
  b.Mv = ws.take<float>(static_cast<size_t>(p.lp) * p.k);
  if (p.sampled) {
    b.Vs = ws.take<float>(static_cast<size_t>(p.n) * p.kq);
    b.P = ws.take<float>(static_cast<size_t>(p.m) * p.kq);
    b.eval2 = ws.take<double>(p.kq);
    b.evec2 = ws.take<float>(static_cast<size_t>(p.kq) * p.kq);
  }
  b.bmax = ws.take<float>(static_cast<size_t>(sign_blocks(p.m)) * p.k);
  b.bidx = ws.take<int64_t>(static_cast<size_t>(sign_blocks(p.m)) * p.k);
  b.sign = ws.take<float>(p.k);
  b.u_hi = ws.take<__nv_bfloat16>(static_cast<size_t>(p.m) * p.kp);
  b.u_lo = ws.take<__nv_bfloat16>(static_cast<size_t>(p.m) * p.kp);
  b.w_hi = ws.take<__nv_bfloat16>(static_cast<size_t>(p.n) * p.kp);
  b.w_lo = ws.take<__nv_bfloat16>(static_cast<size_t>(p.n) * p.kp);
  b.amax = ws.take<unsigned>(3);
  return b;
}

// fp32 -> bf16 hi / lo copies (same leading dimension).
__global__ void split_hilo_kernel(const float* A, int64_t count, __nv_bfloat16* hi, __nv_bfloat16* lo) {
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < count;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float x = A[e];
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    hi[e] = h;
    lo[e] = __float2bfloat16_rn(__fsub_rn(x, __bfloat162float(h)));
  }
}

void launch_split_hilo(const float* A, int64_t count, __nv_bfloat16* hi, __nv_bfloat16* lo, cudaStream_t s) {
  int64_t blocks = (count + 255) / 256;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  split_hilo_kernel<<<static_cast<unsigned>(blocks < 1 ? 1 : blocks), 256, 0, s>>>(A, count, hi, lo);
}

struct Source {             // one matrix seen by the skinny GEMMs (bf16 parts)
  const void* parts[2];
  int nparts;
  int64_t rows, cols, ld;
};

// One pass over `a` (see skinny_gemm.h): Y = A X (mode 0) or A^T X (mode 1),
// written as float32 rows (out) and / or as a transposed bf16 hi / lo copy
// (outT, row stride ldo).
metis_status skinny(const Source& a, int mode, const __nv_bfloat16* xt, int64_t ldx, int xparts, int lp, int cs,
                    float* out, __nv_bfloat16* outT, int64_t ldo, int32_t* dev_status, cudaStream_t s) {
  SkinnyCall c{};
  c.mode = mode;
  c.m = a.rows;
  c.n = a.cols;
  c.lda = a.ld;
  c.A[0] = a.parts[0];
  c.A[1] = a.parts[1];
  c.aparts = a.nparts;
  c.Xt = xt;
  c.ldx = ldx;
  c.xparts = xparts;
  c.lp = lp;
  c.cs = cs;
  c.out = out;
  c.outT = outT;
  c.ldo = ldo;
  c.dev_status = dev_status;
  return run_skinny_gemm(c, s);
}

// CholeskyQR of a rows x lp product the last pass left in b.Y, `passes` times (2 for the only basis
// when there is no power iteration; otherwise 1 for every basis: the Gram is
// float64 from float32 data).  Output: Q (fp32, rows x lp) and Q^T as bf16
// hi / lo rows of qt (row stride ldq).
metis_status cholqr(const SplitBuffers& b, int64_t rows, int lp, float* Q, int64_t ldq, int passes,
                    cudaStream_t s) {
  launch_gram(b.Y, rows, lp, b.gpart, b.G, s);
  METIS_TRY(step_status("cholqr gram"));
  const float* in = b.Y;
  for (int pass = 0; pass < passes; ++pass) {
    const bool last = pass == passes - 1;
    if (!launch_cholesky(b.G, lp, b.Lt, s)) return fail(METIS_ERR_CUDA, "cholqr cholesky shared memory");
    METIS_TRY(step_status("cholqr cholesky"));
    ApplyArgs a{};
    a.in = in;
    a.rows = rows;
    a.kin = lp;
    a.in_ld = lp;
    a.M = b.Lt;
    a.kout = lp;
    a.out = last ? Q : b.Q1;
    a.out_ld = lp;
    if (last) {
      a.outT = b.qt;
      a.lpT = lp;
      a.ldx = ldq;
    } else {
      a.gpart = b.gpart;
    }
    if (!launch_solve(a, s)) return fail(METIS_ERR_CUDA, "cholqr solve");
    METIS_TRY(step_status("cholqr solve"));
    if (!last) {
      launch_gram_reduce(b.gpart, static_cast<int>(apply_blocks(rows)), lp, b.G, s);
      METIS_TRY(step_status("cholqr gram reduce"));
      in = b.Q1;
    }
  }
  return METIS_OK;
}

// Range finder + core on `src` (ms x n): returns Z = src^T Q in b.Zn, Q in
// b.Qm, and the sorted eigen-decomposition of Z^T Z in b.eval / b.evec.
metis_status range_and_core(const SplitPlan& p, const SplitBuffers& b, const Source& src, int power_iters,
                            int max_iters, int32_t* dev_status, cudaStream_t s) {
  const int lp = p.lp;
  if (power_iters > 0) {
    // A^T Y0 spans the same space as A^T orth(Y0): Y0 = A Omega goes to the
    // next product as it is (its hi / lo transpose), and the next basis is
    // orthonormalised
    METIS_TRY(skinny(src, 0, b.omt, p.ld_n, 1, lp, p.cs_m, nullptr, b.qt, p.ld_m, dev_status, s));
  } else {
    METIS_TRY(skinny(src, 0, b.omt, p.ld_n, 1, lp, p.cs_m, b.Y, nullptr, 0, dev_status, s));
    METIS_TRY(cholqr(b, src.rows, lp, b.Qm, p.ld_m, 2, s));
  }
  for (int it = 0; it < power_iters; ++it) {
    METIS_TRY(skinny(src, 1, b.qt, p.ld_m, 2, lp, p.cs_n, b.Y, nullptr, 0, dev_status, s));
    METIS_TRY(cholqr(b, p.n, lp, b.Zn, p.ld_n, 1, s));
    METIS_TRY(skinny(src, 0, b.qt, p.ld_n, 2, lp, p.cs_m2, b.Y, nullptr, 0, dev_status, s));
    // one pass also for the final basis: the Gram is formed in float64 from
    // float32 data, so a pass leaves |Q^T Q - I| near kappa(Y) 2^-23
    METIS_TRY(cholqr(b, src.rows, lp, b.Qm, p.ld_m, 1, s));
  }
  METIS_TRY(skinny(src, 1, b.qt, p.ld_m, 2, lp, p.cs_n, b.Zn, nullptr, 0, dev_status, s));
  launch_gram(b.Zn, p.n, lp, b.gpart, b.G, s);
  METIS_TRY(step_status("core gram"));
  launch_core_eig(b.G, lp, max_iters, b.eval, b.evec, b.eig_ws, dev_status, s);
  return step_status("core eigensolver");
}

metis_status validate_split(const void* A, int dtype, int64_t m, int64_t n, int64_t lda,
                            const metis_split_params* prm, float* U, float* S, float* V, metis_fp4_tensor* U_q,
                            metis_fp4_tensor* V_q, metis_fp4_tensor* R_rows, metis_fp4_tensor* R_cols,
                            int32_t* dev_status) {
  if (!prm || !U || !S || !V || !dev_status) return METIS_ERR_NULL;
  METIS_TRY(validate_dense(A, dtype, m, n, lda));
  if (!valid_fmt(prm->fmt)) return METIS_ERR_ARG;
  if (prm->sketch != METIS_SKETCH_GAUSSIAN && prm->sketch != METIS_SKETCH_SPARSE_SIGN) return METIS_ERR_ARG;
  if (prm->k < 1 || prm->p < 0 || prm->power_iters < 0 || prm->max_core_iters < 1) return METIS_ERR_ARG;
  if (prm->compensate != 0 && prm->compensate != 1) return METIS_ERR_ARG;
  if (prm->compensate && (!U_q || !V_q)) return METIS_ERR_NULL;
  const int l = prm->k + prm->p;
  if (l > 112) return METIS_ERR_SHAPE;
  if (prm->k % 4) return METIS_ERR_SHAPE;  // U, V rows of k floats start on 16-byte boundaries
  if (prm->sample_rows < 0 || prm->sample_rows > m) return METIS_ERR_SHAPE;
  const int64_t ms = prm->sample_rows ? prm->sample_rows : m;
  if (l > ms || l > n) return METIS_ERR_SHAPE;
  if (prm->sketch == METIS_SKETCH_SPARSE_SIGN && (prm->sparse_nnz < 1 || prm->sparse_nnz > 16 || prm->sparse_nnz > l))
    return METIS_ERR_ARG;
  if (m % 32 || n % 32) return METIS_ERR_SHAPE;
  if (m > INT32_MAX || n > INT32_MAX) return METIS_ERR_SHAPE;
  if (U_q) METIS_TRY(check_fp4(U_q, prm->k, m, prm->fmt));
  if (V_q) METIS_TRY(check_fp4(V_q, prm->k, n, prm->fmt));
  if (R_rows) METIS_TRY(check_fp4(R_rows, m, n, prm->fmt));
  if (R_cols) METIS_TRY(check_fp4(R_cols, n, m, prm->fmt));
  return METIS_OK;
}

}  // namespace

}  // namespace metis

using namespace metis;

extern "C" metis_status metis_split(const void* A, int32_t dtype, int64_t m, int64_t n, int64_t lda,
                                    const metis_split_params* prm, float* U, float* S, float* V,
                                    metis_fp4_tensor* U_q, metis_fp4_tensor* V_q, metis_fp4_tensor* R_rows,
                                    metis_fp4_tensor* R_cols, float* R_f32, int32_t* sample_idx, void* workspace,
                                    size_t* workspace_bytes, int32_t* dev_status, void* stream) {
  if (!workspace_bytes) return METIS_ERR_NULL;
  METIS_TRY(validate_split(A, dtype, m, n, lda, prm, U, S, V, U_q, V_q, R_rows, R_cols, dev_status));
  const SplitPlan p = make_plan(m, n, dtype, prm);
  size_t need = 0;
  {
    Carver c(nullptr);
    carve(p, lda, c);
    need = c.used;
    if (U_q) need += quantize_workspace(U_q);
    if (V_q) need += quantize_workspace(V_q);
  }
  if (!workspace) {
    *workspace_bytes = need;
    return METIS_OK;
  }
  if (*workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return METIS_ERR_WORKSPACE;
  if (!device_is_sm100()) return METIS_ERR_UNSUPPORTED;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sms = device_sm_count();
  Carver ws(workspace);
  const SplitBuffers b = carve(p, lda, ws);
  const size_t esz = dtype_size(dtype);

  // the matrix the range finder runs on
  Source full{};
  full.rows = m;
  full.cols = n;
  full.ld = lda;
  Source src = full;
  METIS_TRY(step_status("split entry"));
  if (p.sampled) {
    launch_sample_rows(m, p.ms, prm->seed, b.sel, b.hist, b.idx, sms, s);
    launch_gather_rows(A, n, lda, esz, b.idx, p.ms, b.a_s, s);
    if (sample_idx) cudaMemcpyAsync(sample_idx, b.idx, p.ms * sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
    src.rows = p.ms;
  }
  const void* src_data = p.sampled ? b.a_s : A;
  if (p.fp32) {
    launch_split_hilo(static_cast<const float*>(src_data), src.rows * lda, b.a_hi, b.a_lo, s);
    src.parts[0] = b.a_hi;
    src.parts[1] = b.a_lo;
    src.nparts = 2;
    full.parts[0] = b.a_hi;
    full.parts[1] = b.a_lo;
    full.nparts = 2;
    if (p.sampled) {
      launch_split_hilo(static_cast<const float*>(A), m * lda, b.af_hi, b.af_lo, s);
      full.parts[0] = b.af_hi;
      full.parts[1] = b.af_lo;
    }
  } else {
    src.parts[0] = src_data;
    src.nparts = 1;
    full.parts[0] = A;
    full.nparts = 1;
  }

  if (prm->sketch == METIS_SKETCH_GAUSSIAN)
    launch_gaussian_omega(n, p.l, p.lp, prm->seed, b.omt, p.ld_n, s);
  else
    launch_sparse_sign(n, p.l, p.lp, prm->sparse_nnz, prm->seed, b.omt, p.ld_n, dev_status, s);
  METIS_TRY(step_status("sketch / sampling"));

  const int power_iters = prm->power_iters;
  METIS_TRY(range_and_core(p, b, src, power_iters, prm->max_core_iters, dev_status, s));
  launch_factor_mats(b.eval, b.evec, p.lp, p.k, b.Mu, b.Mv, S, s);
  METIS_TRY(step_status("factor matrices"));

  if (!p.sampled) {
    ApplyArgs au{};
    au.in = b.Qm;
    au.rows = m;
    au.kin = p.lp;
    au.in_ld = p.lp;
    au.M = b.Mu;
    au.kout = p.k;
    au.out = U;
    au.out_ld = p.k;
    au.bmax = b.bmax;   // U's column maxima per 32-row block, for the sign convention
    au.bidx = b.bidx;
    ApplyArgs av{};
    av.in = b.Zn;
    av.rows = n;
    av.kin = p.lp;
    av.in_ld = p.lp;
    av.M = b.Mv;
    av.kout = p.k;
    av.out = V;
    av.out_ld = p.k;
    launch_apply2(au, av, s);
  } else {
    // V_s = Z W_k / sigma (n x k, stored with width kq and as bf16 hi/lo^T)
    cudaMemsetAsync(b.Vs, 0, static_cast<size_t>(n) * p.kq * sizeof(float), s);
    cudaMemsetAsync(b.qt, 0, static_cast<size_t>(2 * p.kq) * p.ld_n * sizeof(__nv_bfloat16), s);
    ApplyArgs avs{};
    avs.in = b.Zn;
    avs.rows = n;
    avs.kin = p.lp;
    avs.in_ld = p.lp;
    avs.M = b.Mv;
    avs.kout = p.k;
    avs.out = b.Vs;
    avs.out_ld = p.kq;
    avs.outT = b.qt;
    avs.lpT = p.kq;
    avs.ldx = p.ld_n;
    launch_apply(avs, s);
    // P = A V_s over all rows, and P^T P
    METIS_TRY(skinny(full, 0, b.qt, p.ld_n, 2, p.kq, skinny_cluster(m, n, sms), b.P, nullptr, 0, dev_status, s));
    launch_gram(b.P, m, p.kq, b.gpart, b.G, s);
    launch_core_eig(b.G, p.kq, prm->max_core_iters, b.eval2, b.evec2, b.eig_ws, dev_status, s);
    launch_factor_mats(b.eval2, b.evec2, p.kq, p.k, b.Mu, b.Mv, S, s);
    ApplyArgs au{};
    au.in = b.P;
    au.rows = m;
    au.kin = p.kq;
    au.in_ld = p.kq;
    au.M = b.Mv;  // U = P W / sigma
    au.kout = p.k;
    au.out = U;
    au.out_ld = p.k;
    au.bmax = b.bmax;
    au.bidx = b.bidx;
    ApplyArgs av{};
    av.in = b.Vs;
    av.rows = n;
    av.kin = p.kq;
    av.in_ld = p.kq;
    av.M = b.Mu;  // V = V_s W
    av.kout = p.k;
    av.out = V;
    av.out_ld = p.k;
    launch_apply2(au, av, s);
  }
  METIS_TRY(step_status("factors"));
  launch_signs_from_blocks(U, m, V, n, p.k, b.bmax, b.bidx, b.sign, s);
  METIS_TRY(step_status("signs"));
  const bool residual = R_rows || R_cols || R_f32;
  cudaMemsetAsync(b.amax, 0, 3 * sizeof(unsigned), s);  // [0] |U|, [1] |V|, [2] |R|
  launch_factor_finish(U, m, V, n, p.k, b.sign, S, p.kp, residual ? b.u_hi : nullptr, b.u_lo, b.w_hi, b.w_lo,
                       b.amax, sms, s);
  METIS_TRY(step_status("factor signs and operands"));
  if (U_q) METIS_TRY(enqueue_quantize(U, METIS_F32, m, p.k, p.k, 0, nullptr, U_q, b.amax, nullptr, ws, s));
  if (V_q) METIS_TRY(enqueue_quantize(V, METIS_F32, n, p.k, p.k, 0, nullptr, V_q, b.amax + 1, nullptr, ws, s));
  if (residual && prm->compensate) {
    // the residual against the factors as quantized: its operands become
    // hi / lo of deq(U_q) and deq(V_q) diag(S)
    auto view = [](const metis_fp4_tensor* t) {
      FactorView f{};
      f.ones = 0;
      f.fmt = t->fmt;
      f.inner = t->inner;
      f.scale_cols = tc_scale_cols(t->fmt, t->inner);
      f.codes = t->codes;
      f.scales = t->scales;
      f.tensor_scale = t->fmt == METIS_NVFP4 ? t->tensor_scale : nullptr;
      return f;
    };
    launch_compensated_operands(view(U_q), view(V_q), m, n, p.k, S, p.kp, b.u_hi, b.u_lo, b.w_hi, b.w_lo, sms, s);
    METIS_TRY(step_status("compensated residual operands"));
  }

  if (residual) {
    ResidualOperands ro{b.u_hi, b.u_lo, b.w_hi, b.w_lo};
    ResidualParams rp{};
    rp.A = A;
    rp.dtype = dtype;
    rp.m = m;
    rp.n = n;
    rp.lda = lda;
    rp.kp = p.kp;
    rp.fmt = prm->fmt;
    rp.amax_bits = b.amax + 2;
    rp.dev_status = dev_status;
    if (prm->fmt == METIS_NVFP4) {
      rp.mode = 0;
      METIS_TRY(run_residual_quant(rp, ro, s));
    }
    rp.mode = 1;
    if (R_rows) {
      cudaMemsetAsync(R_rows->scales, 0, metis_fp4_scales_bytes(prm->fmt, m, n), s);
      rp.r_codes = R_rows->codes;
      rp.r_scales = R_rows->scales;
      rp.r_scale_cols = tc_scale_cols(prm->fmt, n);
      rp.ts_rows = prm->fmt == METIS_NVFP4 ? R_rows->tensor_scale : nullptr;
    }
    if (R_cols) {
      cudaMemsetAsync(R_cols->scales, 0, metis_fp4_scales_bytes(prm->fmt, n, m), s);
      rp.c_codes = R_cols->codes;
      rp.c_scales = R_cols->scales;
      rp.c_scale_cols = tc_scale_cols(prm->fmt, m);
      rp.ts_cols = prm->fmt == METIS_NVFP4 ? R_cols->tensor_scale : nullptr;
    }
    rp.r_tap = R_f32;
    METIS_TRY(run_residual_quant(rp, ro, s));
  }
  return launch_status();
}
