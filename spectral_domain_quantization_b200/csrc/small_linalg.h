// Interface of the small dense linear algebra kernels (small_linalg.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace metis {

struct ApplyArgs {
  const float* in;         // rows x kin, row stride in_ld
  int64_t rows;
  int kin;
  int64_t in_ld;
  const float* M;          // kin x kout, row-major
  int kout;
  float* out;              // optional rows x kout, row stride out_ld
  int64_t out_ld;
  __nv_bfloat16* outT;     // optional [2*lpT][ldx]: hi rows 0..kout-1, lo rows lpT..
  int lpT;
  int64_t ldx;
  double* gpart;           // optional [blocks][kout][kout]
  float* bmax;             // optional [blocks][kout]: max |out| of each 32-row block's columns
  int64_t* bidx;           // with bmax: the first row holding it
};

// row blocks of launch_apply (its Gram partials come one per block)
int64_t apply_blocks(int64_t rows);
// out = in L^-T by forward substitution (M = Lt from launch_cholesky, kin =
// kout = lp, a multiple of 16 up to 112), with the same optional stores as
// launch_apply.  False when the width is not supported or the shared memory
// cannot be granted (nothing is launched).
bool launch_solve(const ApplyArgs& a, cudaStream_t s);
// G = Y^T Y (float64, lp x lp) of a rows x lp float32 Y (row stride lp):
// Gram partials of 32-row blocks (gram_blocks(rows) * lp * lp doubles of
// scratch in gpart), then their sum in block order.
int64_t gram_blocks(int64_t rows);
void launch_gram(const float* Y, int64_t rows, int lp, double* gpart, double* G, cudaStream_t s);
// G = sum of nblocks Gram partials (lp x lp float64 each), in block order.
void launch_gram_reduce(const double* gpart, int nblocks, int lp, double* G, cudaStream_t s);
// Cholesky factor of G = L L^T (lp x lp float64; a pivot below 1e-12 of
// its original diagonal is dropped), for launch_solve: Lt (lp x lp float)
// holds L column by column, Lt[i][i] = 1 / L[i][i] (0 for a dropped pivot) and Lt[i][m] =
// L[m][i] for m > i.  False when the shared memory cannot be granted.
bool launch_cholesky(const double* G, int lp, float* Lt, cudaStream_t s);
void launch_apply(const ApplyArgs& a, cudaStream_t s);
// Two independent products in one launch (blocks of a first, then of b).
void launch_apply2(const ApplyArgs& a, const ApplyArgs& b, cudaStream_t s);
// sign[j] = the sign that makes the largest-|.| entry (lowest row on ties)
// of column j of U positive (applied by launch_factor_finish), from U's
// column maxima per 32-row block that its apply wrote (bmax / bidx).
void launch_signs_from_blocks(float* U, int64_t m, float* V, int64_t n, int k, const float* bmax,
                              const int64_t* bidx, float* sign, cudaStream_t s);
// Symmetric eigen-decomposition of C (n x n float64, n <= 112, a multiple of
// 16), eigenvalues descending in eval, evec[i * n + j] = component i of
// eigenvector j (core_eig.cu).  ws: core_eig_workspace(n) bytes of scratch;
// max_iters caps the multisection rounds per eigenvalue (METIS_DEV_NUMERIC
// when reached).
size_t core_eig_workspace(int n);
void launch_core_eig(double* C, int n, int max_iters, double* eval, float* evec, double* ws, int32_t* dev_status,
                     cudaStream_t s);
void launch_factor_mats(const double* eval, const float* evec, int lp, int k, float* Mu, float* Mv, float* S,
                        cudaStream_t s);
int64_t sign_blocks(int64_t rows);

}  // namespace metis
