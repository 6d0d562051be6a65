/*
 * metis.h -- C ABI of the B200-native spectral-split W4A4G4 linear layer
 * (Metis) and the Averis mean/residual split.
 *
 * What the library computes (sources cited by page title and section):
 *   - "Metis: Training LLMs with FP4 Quantization" (arXiv 2509.00404v4),
 *     abstract and technical framework: the anisotropic spectrum of a weight,
 *     activation or gradient matrix is split into a dominant part and a long
 *     tail that are quantized to FP4 independently (W4A4G4); the split uses
 *     random projection and sparse random sampling to stay cheap.
 *   - SII open-source-week release on Metis, section 2.4 item 1: spectral
 *     decomposition A = U_k S_k V_k^T + R with randomized dimension reduction;
 *     section 2.3 / Fig. 3 and the feature list: block-wise FP4 quantization
 *     (MXFP4, NVFP4) where every block's scale follows the block maximum.
 *   - Retelling of arXiv 2603.10444 (mean bias in FP4 training), Averis
 *     paragraphs: X = 1 mu^T + R with mu the mean over all rows; mean and
 *     residual are quantized separately, in forward and backward.
 *
 * Conventions shared by every entry point
 *   - Memory: the caller owns all memory.  Pointers named "device" must be
 *     device memory of the current CUDA device; "host" pointers are read on the
 *     host before any launch.  The library never allocates, frees, prints or
 *     synchronises the stream; every call only enqueues work on `stream`
 *     (a cudaStream_t; NULL means the legacy default stream).
 *   - Workspace: each call that needs scratch takes `workspace` (device) and
 *     `workspace_bytes` (host, in/out).  With workspace == NULL the call writes
 *     the required size to *workspace_bytes, launches nothing and returns
 *     METIS_OK.  Otherwise *workspace_bytes must be at least that size
 *     (METIS_ERR_WORKSPACE) and the workspace must be 256-byte aligned.  The
 *     workspace is used only during the enqueued work; calls that share one
 *     workspace must be ordered on one stream.
 *   - Errors: argument problems are returned before anything is launched.
 *     Problems found on the device (numerical breakdown, a bounded wait that
 *     expired) are OR-ed into the caller's device word *dev_status as
 *     METIS_DEV_* bits; the caller reads it after synchronising.  dev_status
 *     may be NULL where an entry point says so.
 *   - Layouts: all dense matrices are row-major with a leading dimension in
 *     elements.  FP4 matrices use metis_fp4_tensor below.
 *   - Determinism: identical inputs, sizes and seed give bit-identical outputs
 *     (no atomics on floating-point sums; fixed reduction orders).
 *   - Requires an sm_100 device (B200); METIS_ERR_UNSUPPORTED otherwise.
 */
#ifndef METIS_H
#define METIS_H

#include <stddef.h>
#include <stdint.h>

/* Entry points are the library's only exported symbols (it is built with
 * hidden visibility). */
#if defined(__GNUC__)
#define METIS_API __attribute__((visibility("default")))
#else
#define METIS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  METIS_OK = 0,
  METIS_ERR_NULL = 1,        /* a required pointer is NULL                       */
  METIS_ERR_SHAPE = 2,       /* a size is out of range or not a block multiple   */
  METIS_ERR_ALIGN = 3,       /* a pointer or leading dimension is misaligned     */
  METIS_ERR_UNSUPPORTED = 4, /* not an sm_100 device, or an unsupported option   */
  METIS_ERR_WORKSPACE = 5,   /* workspace too small or misaligned                */
  METIS_ERR_CUDA = 6,        /* a CUDA runtime/driver call failed                */
  METIS_ERR_ARG = 7          /* any other invalid argument (enum value, k, ...)  */
} metis_status;

/* bits OR-ed into *dev_status by kernels */
#define METIS_DEV_NUMERIC 1  /* the core eigensolver hit max_core_iters          */
#define METIS_DEV_TIMEOUT 2  /* a bounded device wait expired; outputs invalid   */
#define METIS_DEV_SAMPLING 4 /* a sparse-sign row could not draw its columns     */

typedef enum { METIS_BF16 = 0, METIS_F32 = 1 } metis_dtype;
typedef enum { METIS_MXFP4 = 0, METIS_NVFP4 = 1 } metis_fp4_fmt;
typedef enum { METIS_SKETCH_GAUSSIAN = 0, METIS_SKETCH_SPARSE_SIGN = 1 } metis_sketch;

/*
 * One FP4 matrix, "outer x inner", blocks of 32 (MXFP4) or 16 (NVFP4)
 * consecutive elements along `inner`.  A GEMM operand is stored with `inner`
 * equal to the contraction dimension ("K-major").
 *
 *   codes          device, outer * inner / 2 bytes, row-major [outer][inner/2];
 *                  element 2j in the low nibble of byte j.  E2M1 code
 *                  s|e1 e0|m: magnitudes {0,.5,1,1.5,2,3,4,6}.
 *   scales         device, metis_fp4_scales_bytes(fmt, outer, inner) bytes:
 *                  the tensor-core layout.  Rows are padded to 128 and scale
 *                  columns to a whole 256-element K tile; scale (r, c) sits at
 *                  byte ((r/128)*(C/4) + c/4)*512 + (r%32)*16 + ((r%128)/32)*4
 *                  + c%4 where C is the padded scale-column count.  Padding is
 *                  zero.  MXFP4: E8M0 codes (2^(code-127)).  NVFP4: E4M3 codes.
 *   scales_linear  device, optional (may be NULL): [outer][inner/bs] codes.
 *   tensor_scale   device, one float: NVFP4 decode scale s_t (value =
 *                  e2m1 * e4m3 * s_t).  Written by the quantizer.  Ignored for
 *                  MXFP4 (may be NULL).
 *   inner_sum      device, optional (may be NULL): one float per outer index,
 *                  the sum over `inner` of the dequantized values (float32,
 *                  fixed summation order).
 */
typedef struct {
  int32_t fmt;          /* metis_fp4_fmt */
  int64_t outer;
  int64_t inner;
  uint8_t* codes;
  uint8_t* scales;
  uint8_t* scales_linear;
  float* tensor_scale;
  float* inner_sum;
} metis_fp4_tensor;

/* Host-only helpers (no device work): buffer sizes for a metis_fp4_tensor. */
METIS_API size_t metis_fp4_codes_bytes(int64_t outer, int64_t inner);
METIS_API size_t metis_fp4_scales_bytes(int32_t fmt, int64_t outer, int64_t inner);

/* Host-only: short description of a status code (static string). */
METIS_API const char* metis_status_string(int32_t status);

/* Host-only: 1 if a device of compute capability 10.x is current, else 0. */
METIS_API int32_t metis_device_supported(void);

/* Host-only: description of the last METIS_ERR_CUDA reported on this thread
 * (which step failed and the CUDA error string); "" if none.  The string is
 * owned by the library and overwritten by the next failure on the thread. */
METIS_API const char* metis_last_error(void);

/*
 * metis_selftest_wait_timeout -- check of the failure detection every kernel
 * relies on.  One thread runs the library's bounded barrier wait on a phase
 * that nothing completes, with a limit of limit_ns (1 .. 1e9 ns), and must
 * OR METIS_DEV_TIMEOUT into *dev_status (device int32, caller-owned) and
 * return.  The pages have no counterpart: this is the library's own check
 * that a stalled wait ends with a status instead of hanging.
 * Errors: METIS_ERR_NULL (dev_status), METIS_ERR_ARG (limit out of range),
 * METIS_ERR_UNSUPPORTED (no sm_100 device), METIS_ERR_CUDA (launch).
 */
METIS_API metis_status metis_selftest_wait_timeout(uint64_t limit_ns, int32_t* dev_status, void* stream);

/*
 * metis_quantize_fp4 -- block-quantize a dense matrix to FP4.
 * Source: SII release section 2.3 / Fig. 3 (one scale per block, set by the
 * block maximum) and the feature list (MXFP4 / NVFP4).  Bit-level rules
 * (OCP MX v1.0 for MXFP4; two-level NVFP4):
 *   MXFP4 (block 32): a = max|x|; a == 0 -> scale code 0, codes 0; else
 *     se = clamp(floor(log2 a) - 2, -127, 127), scale code se + 127,
 *     code = E2M1(x * 2^-se).
 *   NVFP4 (block 16): alpha = max|x| over the tensor; s_t = alpha / 2688
 *     (1 if alpha == 0); t = (a / s_t) / 6; d = E4M3(t) round-to-nearest-even,
 *     saturating at 448; d == 0 -> codes 0; else code = E2M1(x * (1/(d*s_t))).
 *   E2M1 rounds to nearest, ties to the even code, saturates at 6; the sign bit
 *   is the sign of the scaled value.  All arithmetic is IEEE float32 in this
 *   order (bit-exact against the CPU oracle).
 *
 *   X            device, rows x cols, leading dimension ld (elements),
 *                dtype METIS_BF16 or METIS_F32.  16-byte aligned rows.
 *   block_axis   1: blocks along cols (out->outer = rows, out->inner = cols);
 *                0: blocks along rows (out->outer = cols, out->inner = rows).
 *   sub_col      device, optional: cols floats; the quantized value is
 *                fl32(x_ij - sub_col[j]) (the Averis residual).  May be NULL.
 *   out          host struct with device buffers; out->fmt selects the format;
 *                outer/inner must match.  The blocked dimension must be a
 *                multiple of 32 (METIS_ERR_SHAPE).
 * Workspace: NVFP4 needs a few bytes for the tensor maximum.
 */
METIS_API metis_status metis_quantize_fp4(const void* X, int32_t dtype, int64_t rows, int64_t cols,
                                int64_t ld, int32_t block_axis, const float* sub_col,
                                metis_fp4_tensor* out, void* workspace,
                                size_t* workspace_bytes, void* stream);

/*
 * metis_quantize_fp4_noalloc -- metis_quantize_fp4 for callers that cannot
 * provide scratch memory.  (No counterpart in the source pages: this is a
 * library convenience, not part of the method.)
 *
 * Who needs it: code that may not allocate device memory where it quantizes
 * (a runtime that owns every device byte through its own arena, a plugin whose
 * host framework forbids allocation while it runs, a loop that must not block
 * on the allocator) or a program that simply has no spare device buffer.
 *
 * It takes the same arguments as metis_quantize_fp4 minus the workspace and
 * produces identical bytes.  Its scratch (the NVFP4 tensor-maximum word and,
 * when out->inner_sum is set, outer * ceil(inner / 64) partial sums) lives in
 * one fixed array of metis_noalloc_scratch_bytes() (2 MiB) compiled into the
 * library; every GPU that loads the library keeps that array until the
 * process exits.  Larger requests return METIS_ERR_WORKSPACE (see
 * metis_last_error()); use metis_quantize_fp4 for them.
 *   - The first call on a device looks up the array's device address (this may
 *     load the library's device code); make that first call before any CUDA
 *     stream capture.  The address is kept per device and context: after the
 *     context is destroyed and re-created (cudaDeviceReset), the next call
 *     looks it up again, so make that call before any capture too.
 *   - All calls share the one array: calls whose GPU work overlaps (different
 *     streams, concurrent host threads) race and must be ordered by the caller.
 *     The call zeroes what must start at zero itself.
 * The function never calls cudaMalloc, cudaFree or any allocating routine.
 */
METIS_API metis_status metis_quantize_fp4_noalloc(const void* X, int32_t dtype, int64_t rows, int64_t cols,
                                        int64_t ld, int32_t block_axis, const float* sub_col,
                                        metis_fp4_tensor* out, void* stream);

/* Host-only: size in bytes of the fixed scratch array of the _noalloc call. */
METIS_API size_t metis_noalloc_scratch_bytes(void);

/*
 * Parameters of the randomized split (host struct).
 *   k, p          rank kept (a multiple of 4) and oversampling; l = k + p <= 112,
 *                 l <= min(m, n)
 *                 (or <= sample_rows), l a multiple of 16 is not required.
 *   power_iters   q >= 0 subspace iterations.
 *   seed          Philox4x32-10 key for the sketch and the row sample.
 *   sketch        METIS_SKETCH_GAUSSIAN or METIS_SKETCH_SPARSE_SIGN.
 *   sparse_nnz    nonzeros per input coordinate of the sparse-sign sketch.
 *   sample_rows   0, or the number of rows sampled to find the right singular
 *                 subspace (then power_iters applies to the sample).
 *   fmt           metis_fp4_fmt of every quantized output.
 *   max_core_iters  cap on the multisection rounds that find each eigenvalue
 *                 of the core Gram (about 11 are needed; 64 is a safe
 *                 value); reaching it sets METIS_DEV_NUMERIC in *dev_status.
 *   compensate    0: R = A - U diag(S) V^T with the float32 factors (the
 *                 pages' split).  1: the error-compensated residual
 *                 R = A - deq(U_q) diag(S) deq(V_q)^T, formed from the FP4
 *                 factors as quantized, so that the quantized residual also
 *                 absorbs the factors' quantization error; needs U_q and V_q
 *                 (METIS_ERR_NULL otherwise).  Zero-initialise the struct
 *                 to get 0.
 */
typedef struct {
  int32_t k;
  int32_t p;
  int32_t power_iters;
  uint64_t seed;
  int32_t sketch;
  int32_t sparse_nnz;
  int64_t sample_rows;
  int32_t fmt;
  int32_t max_core_iters;
  int32_t compensate;
} metis_split_params;

/*
 * metis_split -- spectral split A = U diag(S) V^T + R and FP4 quantization of
 * U, V and R.
 * Source: SII release section 2.4 item 1 (dominant + long-tail split with
 * randomized dimension reduction); "Metis: Training LLMs with FP4
 * Quantization" abstract (random projection and sparse random sampling);
 * older Metis abstract item (i) (random embedding).
 * Steps: [sample rows] -> Omega (Philox Gaussian / sparse sign, bf16) ->
 * Y = A Omega -> q x (A^T Y, CholeskyQR, A Q, CholeskyQR) (with q = 0 a
 * two-pass CholeskyQR of Y) -> Z = A^T Q -> eigen-decomposition of the l x l
 * core Gram C = Z^T Z in float64 (Householder tridiagonalisation, multisection
 * on Sturm counts, eigenvectors from the twisted factorisation) -> top k,
 * U = Q W, V = Z W S^-1, signs (largest-|.| entry of each U column made
 * positive) -> R = A - U S V^T (or, with compensate, A minus the product of
 * the dequantized FP4 factors) fused with FP4 quantization.
 * With sample_rows > 0: V_s from the sampled rows, P = A V_s, the
 * eigen-decomposition P^T P = W diag(sigma^2) W^T with the same solver (the SVD
 * of P's triangular QR factor in exact arithmetic); U = P W / sigma,
 * V = V_s W.
 *
 *   A, dtype, m, n, lda   device input (bf16 or f32), row-major, 16-byte rows.
 *   U       device m x k float (row-major), S device k floats (descending),
 *   V       device n x k float.
 *   U_q     optional FP4 of U quantized along m (outer = k, inner = m).
 *   V_q     optional FP4 of V quantized along n (outer = k, inner = n).
 *   R_rows  optional FP4 of R with blocks along n (outer = m, inner = n).
 *   R_cols  optional FP4 of R with blocks along m (outer = n, inner = m).
 *   R_f32   optional device m x n float tap of the residual the quantizer saw.
 *   sample_idx  optional device int32[sample_rows]: the sampled rows.
 *   dev_status  device int32 (required).
 * Quantized outputs need m and n multiples of 32 along their blocked axis.
 * Sketch tap: after the call, in stream order, the first lp * round_up(n, 8)
 * bf16 values of the workspace hold Omega^T (lp = round_up(k + p, 16) rows of
 * round_up(n, 8) entries, row j = column j of Omega; rows past k + p and
 * entries past n are zero).  It is read-only output for tests; the rest of
 * the workspace is scratch.
 */
METIS_API metis_status metis_split(const void* A, int32_t dtype, int64_t m, int64_t n, int64_t lda,
                         const metis_split_params* prm, float* U, float* S, float* V,
                         metis_fp4_tensor* U_q, metis_fp4_tensor* V_q,
                         metis_fp4_tensor* R_rows, metis_fp4_tensor* R_cols, float* R_f32,
                         int32_t* sample_idx, void* workspace, size_t* workspace_bytes,
                         int32_t* dev_status, void* stream);

/*
 * One operand of an FP4 product C = A B (host struct):
 *   left  operand A (M x K) = R + F diag(S) P^T
 *   right operand B (K x N) = R + P diag(S) F^T
 *   R  FP4, quantized along the contraction axis: outer = M (left) or N
 *      (right), inner = K.  Required.
 *   k  rank of the low-rank term (0 = plain FP4 operand; then P, F, S unused).
 *   P  FP4, the factor along the contraction axis: outer = k, inner = K.
 *      NULL means the all-ones vector (k must be 1).
 *   F  FP4, the factor along the free axis: outer = k, inner = M or N.
 *      NULL means the all-ones vector (k must be 1).
 *   S  device k floats (NULL = all ones).
 * Averis operands are rank 1 with one factor all-ones; the product then needs
 * R->inner_sum of the other operand's residual where the ones-vector is
 * contracted against it.  Both operands must share one FP4 format.
 */
typedef struct {
  const metis_fp4_tensor* R;
  int32_t k;
  const metis_fp4_tensor* P;
  const metis_fp4_tensor* F;
  const float* S;
  /* bit 0 (METIS_REQUANT_LOWRANK): re-quantize to FP4 the low-rank
   * intermediate formed from this operand's factors (T1 for a right operand,
   * T2 for a left operand), in blocks along its k, before it enters the
   * product.  0 keeps it in float32 (bf16 hi/lo).  Other bits: 0. */
  int32_t flags;
} metis_operand;

#define METIS_REQUANT_LOWRANK 1

/*
 * metis_linear_fwd -- Y = X W on FP4 operands (W4A4 forward).
 * Source: "Metis: Training LLMs with FP4 Quantization" abstract (W4A4G4);
 * SII release section 2.4 item 1 (both parts of the split take part).
 * Computes Y = R_X R_W (block-scaled tcgen05 FP4 MMA, fp32 accumulation) plus
 * the low-rank terms T1 F_W^T + F_X T2 accumulated into the same tensor-memory
 * accumulator (T1 = (R_X P_W + F_X S_X P_X^T P_W) S_W, T2 = S_X P_X^T R_W).
 *   X  left operand (M x K), W right operand (K x N).
 *   Y  device M x N, y_dtype METIS_F32 or METIS_BF16, leading dimension ldy.
 * K must be a multiple of 32, and M, N, K at most INT32_MAX (METIS_ERR_SHAPE).
 */
METIS_API metis_status metis_linear_fwd(const metis_operand* X, const metis_operand* W, int64_t M,
                              int64_t N, int64_t K, void* Y, int32_t y_dtype, int64_t ldy,
                              void* workspace, size_t* workspace_bytes, int32_t* dev_status,
                              void* stream);

/*
 * metis_linear_bwd -- the two backward products of Y = X W on FP4 operands:
 *   dX = dY W^T  (left operand dY_n: dY quantized along N;
 *                 right operand Wt:  W quantized along N, P = V_W, F = U_W)
 *   dW = X^T dY  (left operand Xt:   X quantized along M, P = U_X, F = V_X;
 *                 right operand dY_m: dY quantized along M)
 * Source: "Metis: Training LLMs with FP4 Quantization" abstract (FP4
 * gradients, G4); Averis paragraphs (the output gradient is split too).
 *   dX  device M x K (or NULL to skip), dW device K x N (or NULL to skip),
 *   out_dtype METIS_F32 or METIS_BF16; ld_dx, ld_dw leading dimensions.
 * N must be a multiple of 32 for dX and M a multiple of 32 for dW; M, N and
 * K are at most INT32_MAX (METIS_ERR_SHAPE).
 */
METIS_API metis_status metis_linear_bwd(const metis_operand* dY_n, const metis_operand* Wt,
                              const metis_operand* Xt, const metis_operand* dY_m, int64_t M,
                              int64_t N, int64_t K, void* dX, int64_t ld_dx, void* dW,
                              int64_t ld_dw, int32_t out_dtype, void* workspace,
                              size_t* workspace_bytes, int32_t* dev_status, void* stream);

/*
 * averis_split -- X = 1 mu^T + R with mu the mean over all rows, then FP4 of
 * mu and R.
 * Source: retelling of arXiv 2603.10444, Averis paragraphs (mean over all
 * rows, broadcast subtraction, separate quantization of mean and residual;
 * the same split is applied to the output gradient in the backward pass).
 *   X, dtype, m, n, ld  device input.
 *   mean     device n floats: mu_j = (sum_i x_ij) / m (float32, fixed order).
 *   mean_q   optional FP4 of mu (outer = 1, inner = n).
 *   R_rows   optional FP4 of fl32(x_ij - mu_j), blocks along n (outer m).
 *   R_cols   optional FP4 of the same residual, blocks along m (outer n).
 *   R_f32    optional device m x n float tap.
 * NVFP4 takes the residual's tensor maximum from the column minima and maxima
 * (exact: rounding is monotonic), so X is read once for the statistics and
 * once per requested residual axis.  dev_status (device int32, may be NULL):
 * a bounded wait of the TMA-fed bf16 kernels that gives up ORs in
 * METIS_DEV_TIMEOUT.
 */
METIS_API metis_status averis_split(const void* X, int32_t dtype, int64_t m, int64_t n, int64_t ld,
                          int32_t fmt, float* mean, metis_fp4_tensor* mean_q,
                          metis_fp4_tensor* R_rows, metis_fp4_tensor* R_cols, float* R_f32,
                          void* workspace, size_t* workspace_bytes, int32_t* dev_status,
                          void* stream);

/*
 * metis_spectral_scale -- adaptive spectral learning: the gradient G of a
 * split weight W = U diag(S) V^T + R preconditioned along W's singular
 * directions.
 * Source: SII release section 2.4 item 2 (the gradients along the mid and
 * low singular-value directions are scaled up by an inverse normalisation,
 * so that long-tail directions keep learning, without amplifying noise);
 * older Metis abstract item (ii) (adaptive learning rates in the spectral
 * domain).  The pages give no formula; the reading taken is
 *   lambda_i = min(S_1 / S_i, cap)   (1 where S_i <= 0),
 *   G' = (I + U (L - I) U^T) G (I + V (L - I) V^T),  L = diag(sqrt(lambda)),
 * so the component along u_i v_j^T is scaled by sqrt(lambda_i lambda_j), a
 * component with one side in a split direction by that side's
 * sqrt(lambda), and the rest of G (the long tail) is left as it is.
 *   G, K, N, ldg  device float32 gradient, row-major, 16-byte rows.
 *   U, S, V       device float32 factors of the split of W (K x k, k, N x k),
 *                 as metis_split writes them (orthonormal columns, S
 *                 descending).
 *   k             1 .. 64.  cap >= 1.
 *   Gout          device K x N float32 (row stride N, 16-byte aligned); may
 *                 not alias G.
 * K and N must be multiples of 32 (METIS_ERR_SHAPE).  The rank-2k update is
 * formed with bf16 hi / lo tensor-core products, so G' carries a relative
 * error of about 2^-16 of the update on top of float32 rounding.
 */
METIS_API metis_status metis_spectral_scale(const float* G, int64_t K, int64_t N, int64_t ldg,
                                  const float* U, const float* S, const float* V, int32_t k,
                                  float cap, float* Gout, void* workspace, size_t* workspace_bytes,
                                  int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* METIS_H */
