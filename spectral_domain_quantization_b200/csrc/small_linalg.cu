// Small dense linear algebra of the randomized split (l = k + p <= 128):
// Gram matrices, Cholesky with rank drop, triangular inverse (CholeskyQR),
// row-block products, the Jacobi eigensolver of the core, factor assembly and
// the sign convention.
//
// Source: SII release on Metis, section 2.4 item 1 (spectral decomposition in
// a low-dimensional space after randomized reduction); older Metis abstract
// item (i) (random embedding separates dominant from long-tail parts).
//
// Numerics: Gram matrices are accumulated in float64 from float32 rows;
// Cholesky, the triangular inverse and Jacobi run in float64 in one CTA's
// shared memory; tall row blocks are multiplied in float32.
//   * CholeskyQR: G = Y^T Y = L L^T, Q = Y L^-T.  A pivot that falls below
//     1e-12 of its original diagonal (a numerically dependent sketch column,
//     e.g. for an exactly low-rank input) is dropped: that column of Q
//     becomes zero instead of amplified rounding noise.
//   * Core SVD via one-sided Jacobi of B^T, carried out on its l x l Gram
//     C = B B^T (rotations chosen from the Gram entries, as one-sided Jacobi
//     does): C = W diag(sigma^2) W^T, then U = Q W_k, V = B^T W_k / sigma.
//     Rotations use the parallel (round-robin) ordering: l/2 disjoint pairs
//     per step, l-1 steps per sweep.
#include "common.cuh"
#include "abi_common.h"
#include "small_linalg.h"

namespace metis {

namespace {

constexpr int kRowsPerBlock = 32;
constexpr double kDropTol = 1e-12;

// Gram partial of a row block held in shared memory (rows x cols floats with
// row stride ld): out[i][j] for all i, j (full symmetric matrix).
MDEV void gram_block(const float* ys, int rows, int cols, int ld, double* out) {
  const int n = cols * cols;
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const int i = e / cols, j = e - i * cols;
    if (j < i) continue;
    double acc = 0.0;
    for (int r = 0; r < rows; ++r) acc += static_cast<double>(ys[r * ld + i]) * static_cast<double>(ys[r * ld + j]);
    out[i * cols + j] = acc;
    out[j * cols + i] = acc;
  }
}

// Sum split partials into Y (optional) and the Gram partial of each block.
__global__ void gram_kernel(const float* partial, int splits, int64_t rows, int lp, float* Y, double* gpart) {
  extern __shared__ float ys[];  // kRowsPerBlock x (lp + 1)
  const int ld = lp + 1;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kRowsPerBlock;
  const int nr = static_cast<int>(imin64(kRowsPerBlock, rows - r0));
  for (int e = threadIdx.x; e < kRowsPerBlock * lp; e += blockDim.x) {
    const int r = e / lp, c = e - r * lp;
    float v = 0.f;
    if (r < nr) {
      for (int s = 0; s < splits; ++s) v += partial[(static_cast<int64_t>(s) * rows + r0 + r) * lp + c];
      if (Y) Y[(r0 + r) * lp + c] = v;
    }
    ys[r * ld + c] = v;
  }
  __syncthreads();
  gram_block(ys, nr, lp, ld, gpart + static_cast<int64_t>(blockIdx.x) * lp * lp);
}

__global__ void gram_reduce_kernel(const double* gpart, int nblocks, int n2, double* G) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n2) return;
  double s = 0.0;
  for (int b = 0; b < nblocks; ++b) s += gpart[static_cast<int64_t>(b) * n2 + e];
  G[e] = s;
}

// G = L L^T (with drops), then Rinv = L^-T (upper triangular, float32).
__global__ void cholesky_inv_kernel(const double* G, int lp, float* Rinv) {
  extern __shared__ double sm[];
  const int ld = lp + 1;
  double* L = sm;                  // lp x ld
  double* X = L + lp * ld;         // lp x ld, becomes L^-1
  double* diag0 = X + lp * ld;     // lp
  double* invd = diag0 + lp;       // lp
  const int t = threadIdx.x, nt = blockDim.x;
  for (int e = t; e < lp * lp; e += nt) {
    const int i = e / lp, j = e - i * lp;
    L[i * ld + j] = G[e];
    X[i * ld + j] = i == j ? 1.0 : 0.0;
  }
  __syncthreads();
  for (int i = t; i < lp; i += nt) diag0[i] = L[i * ld + i];
  __syncthreads();
  for (int j = 0; j < lp; ++j) {
    if (t == 0) {
      const double d = L[j * ld + j];
      const bool drop = !(diag0[j] > 0.0) || !(d > kDropTol * diag0[j]);
      const double piv = drop ? 0.0 : sqrt(d);
      invd[j] = drop ? 0.0 : 1.0 / piv;
      L[j * ld + j] = piv;
    }
    __syncthreads();
    const double inv = invd[j];
    for (int i = j + 1 + t; i < lp; i += nt) L[i * ld + j] *= inv;
    __syncthreads();
    const int w = lp - j - 1;
    for (int e = t; e < w * w; e += nt) {
      const int i = j + 1 + e / w, c = j + 1 + e % w;
      if (c <= i) L[i * ld + c] -= L[i * ld + j] * L[c * ld + j];
    }
    __syncthreads();
  }
  // forward substitution for X = L^-1, one row at a time
  for (int k = 0; k < lp; ++k) {
    const double inv = invd[k];
    for (int c = t; c <= k; c += nt) X[k * ld + c] *= inv;
    __syncthreads();
    const int rows = lp - k - 1, cols = k + 1;
    for (int e = t; e < rows * cols; e += nt) {
      const int i = k + 1 + e / cols, c = e % cols;
      X[i * ld + c] -= L[i * ld + k] * X[k * ld + c];
    }
    __syncthreads();
  }
  for (int e = t; e < lp * lp; e += nt) {
    const int j = e / lp, c = e - j * lp;  // Rinv[j][c] = X[c][j]
    Rinv[e] = c >= j ? static_cast<float>(X[c * ld + j]) : 0.f;
  }
}

// out = in (rows x kin, row stride in_ld) * Mx (kin x kout, row-major).
// Optional: fp32 out (row stride out_ld), transposed bf16 hi/lo copy
// outT[c][row] and outT[lp + c][row] (row stride ldx), Gram partial.
__global__ void apply_kernel(ApplyArgs a) {
  extern __shared__ float smf[];
  float* Ms = smf;                                     // kin x kout
  float* In = Ms + a.kin * a.kout;                     // kRowsPerBlock x (kin + 1)
  float* Out = In + kRowsPerBlock * (a.kin + 1);       // kRowsPerBlock x (kout + 1)
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kRowsPerBlock;
  const int nr = static_cast<int>(imin64(kRowsPerBlock, a.rows - r0));
  for (int e = threadIdx.x; e < a.kin * a.kout; e += blockDim.x) Ms[e] = a.M[e];
  for (int e = threadIdx.x; e < kRowsPerBlock * a.kin; e += blockDim.x) {
    const int r = e / a.kin, c = e - r * a.kin;
    In[r * (a.kin + 1) + c] = r < nr ? a.in[(r0 + r) * a.in_ld + c] : 0.f;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kRowsPerBlock * a.kout; e += blockDim.x) {
    const int c = e / kRowsPerBlock, r = e - c * kRowsPerBlock;  // row fastest
    float acc = 0.f;
    const int j0 = a.upper ? 0 : 0;
    const int j1 = a.upper ? c + 1 : a.kin;
    for (int j = j0; j < j1; ++j) acc = fmaf(In[r * (a.kin + 1) + j], Ms[j * a.kout + c], acc);
    Out[r * (a.kout + 1) + c] = acc;
    if (r < nr) {
      if (a.out) a.out[(r0 + r) * a.out_ld + c] = acc;
      if (a.outT) {
        const __nv_bfloat16 hi = __float2bfloat16_rn(acc);
        const __nv_bfloat16 lo = __float2bfloat16_rn(__fsub_rn(acc, __bfloat162float(hi)));
        a.outT[static_cast<int64_t>(c) * a.ldx + r0 + r] = hi;
        a.outT[static_cast<int64_t>(a.lpT + c) * a.ldx + r0 + r] = lo;
      }
    }
  }
  if (a.gpart) {
    __syncthreads();
    gram_block(Out, nr, a.kout, a.kout + 1, a.gpart + static_cast<int64_t>(blockIdx.x) * a.kout * a.kout);
  }
}

// Round-robin pairing: in step r of a sweep over n (even) indices, slot i
// pairs with slot n-1-i; slot 0 holds index 0, slots 1..n-1 rotate.
MDEV int rr_index(int slot, int step, int n) {
  if (slot == 0) return 0;
  return ((slot - 1 + step) % (n - 1)) + 1;
}

// Symmetric Jacobi eigen-decomposition of C (n x n float64, n even), sorted
// descending.  evec[i * n + j] = component i of eigenvector j.
__global__ void jacobi_kernel(const double* C, int n, int max_sweeps, double tol, double* eval, float* evec,
                              int32_t* dev_status) {
  extern __shared__ double sd[];
  const int ld = n + 1;
  double* A = sd;              // n x ld
  double* V = A + n * ld;      // n x ld
  double* cs = V + n * ld;     // n/2 cosines
  double* sn = cs + n / 2;     // n/2 sines
  double* red = sn + n / 2;    // blockDim reduction scratch
  __shared__ int pairs_p[64], pairs_q[64];
  __shared__ int stop;
  const int t = threadIdx.x, nt = blockDim.x;
  const int half = n / 2;
  for (int e = t; e < n * n; e += nt) {
    const int i = e / n, j = e - i * n;
    A[i * ld + j] = C[e];
    V[i * ld + j] = i == j ? 1.0 : 0.0;
  }
  if (t == 0) stop = 0;
  __syncthreads();
  // total squared norm (for the relative stopping rule)
  double tot = 0.0;
  for (int e = t; e < n * n; e += nt) {
    const double v = A[(e / n) * ld + e % n];
    tot += v * v;
  }
  red[t] = tot;
  __syncthreads();
  for (int w = nt / 2; w > 0; w >>= 1) {
    if (t < w) red[t] += red[t + w];
    __syncthreads();
  }
  const double total = red[0];
  __syncthreads();
  int sweep = 0;
  for (; sweep < max_sweeps; ++sweep) {
    // off-diagonal norm
    double off = 0.0;
    for (int e = t; e < n * n; e += nt) {
      const int i = e / n, j = e - i * n;
      if (i != j) off += A[i * ld + j] * A[i * ld + j];
    }
    red[t] = off;
    __syncthreads();
    for (int w = nt / 2; w > 0; w >>= 1) {
      if (t < w) red[t] += red[t + w];
      __syncthreads();
    }
    if (t == 0) stop = !(red[0] > tol * tol * total);
    __syncthreads();
    if (stop) break;
    for (int step = 0; step < n - 1; ++step) {
      if (t < half) {
        int p = rr_index(t, step, n), q = rr_index(n - 1 - t, step, n);
        if (p > q) {
          const int x = p;
          p = q;
          q = x;
        }
        pairs_p[t] = p;
        pairs_q[t] = q;
        const double apq = A[p * ld + q];
        double c = 1.0, s = 0.0;
        if (apq != 0.0) {
          const double theta = (A[q * ld + q] - A[p * ld + p]) / (2.0 * apq);
          const double tt = (theta >= 0.0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(1.0 + theta * theta));
          c = 1.0 / sqrt(1.0 + tt * tt);
          s = tt * c;
        }
        cs[t] = c;
        sn[t] = s;
      }
      __syncthreads();
      // columns p, q of A and V
      for (int e = t; e < half * n; e += nt) {
        const int k = e / n, i = e - k * n;
        const int p = pairs_p[k], q = pairs_q[k];
        const double c = cs[k], s = sn[k];
        const double aip = A[i * ld + p], aiq = A[i * ld + q];
        A[i * ld + p] = c * aip - s * aiq;
        A[i * ld + q] = s * aip + c * aiq;
        const double vip = V[i * ld + p], viq = V[i * ld + q];
        V[i * ld + p] = c * vip - s * viq;
        V[i * ld + q] = s * vip + c * viq;
      }
      __syncthreads();
      // rows p, q of A
      for (int e = t; e < half * n; e += nt) {
        const int k = e / n, j = e - k * n;
        const int p = pairs_p[k], q = pairs_q[k];
        const double c = cs[k], s = sn[k];
        const double apj = A[p * ld + j], aqj = A[q * ld + j];
        A[p * ld + j] = c * apj - s * aqj;
        A[q * ld + j] = s * apj + c * aqj;
      }
      __syncthreads();
    }
  }
  if (t == 0 && sweep >= max_sweeps) report(dev_status, METIS_DEV_NUMERIC);
  // sort descending (ties: lower index first)
  for (int j = t; j < n; j += nt) {
    const double lj = A[j * ld + j];
    int rank = 0;
    for (int i = 0; i < n; ++i) {
      const double li = A[i * ld + i];
      rank += (li > lj) || (li == lj && i < j);
    }
    eval[rank] = lj;
    for (int i = 0; i < n; ++i) evec[i * n + rank] = static_cast<float>(V[i * ld + j]);
  }
}

// Factor matrices from the sorted eigen-decomposition of the core Gram:
// Mu = W_k (lp x k), Mv = W_k diag(1/sigma) (0 where sigma is negligible),
// S = sigma_k.
__global__ void factor_mats_kernel(const double* eval, const float* evec, int lp, int k, float* Mu, float* Mv,
                                   float* S) {
  const double top = eval[0] > 0.0 ? sqrt(eval[0]) : 0.0;
  for (int e = threadIdx.x; e < lp * k; e += blockDim.x) {
    const int i = e / k, j = e - i * k;
    const double ev = eval[j];
    const double sigma = ev > 0.0 ? sqrt(ev) : 0.0;
    const float w = evec[i * lp + j];
    Mu[e] = w;
    Mv[e] = (sigma > 1e-12 * top && sigma > 0.0) ? static_cast<float>(w / sigma) : 0.f;
  }
  for (int j = threadIdx.x; j < k; j += blockDim.x) {
    const double ev = eval[j];
    S[j] = static_cast<float>(ev > 0.0 ? sqrt(ev) : 0.0);
  }
}

// Per row block: for each column, the largest |U| and its lowest row index.
__global__ void colmax_kernel(const float* U, int64_t rows, int k, float* bmax, int64_t* bidx) {
  const int j = threadIdx.x;
  if (j >= k) return;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * 256;
  float best = -1.f;
  int64_t bi = 0;
  for (int64_t r = r0; r < imin64(r0 + 256, rows); ++r) {
    const float v = fabsf(U[r * k + j]);
    if (v > best) {
      best = v;
      bi = r;
    }
  }
  bmax[static_cast<int64_t>(blockIdx.x) * k + j] = best;
  bidx[static_cast<int64_t>(blockIdx.x) * k + j] = bi;
}

__global__ void sign_kernel(const float* U, const float* bmax, const int64_t* bidx, int nblocks, int k, float* sign) {
  const int j = threadIdx.x;
  if (j >= k) return;
  float best = -1.f;
  int64_t bi = 0;
  for (int b = 0; b < nblocks; ++b) {
    const float v = bmax[static_cast<int64_t>(b) * k + j];
    if (v > best) {
      best = v;
      bi = bidx[static_cast<int64_t>(b) * k + j];
    }
  }
  sign[j] = U[bi * k + j] < 0.f ? -1.f : 1.f;
}

__global__ void flip_kernel(float* X, int64_t rows, int k, const float* sign) {
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < rows * k;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x)
    X[e] *= sign[e % k];
}

int blocks(int64_t n, int sms) {
  int64_t b = (n + 255) / 256;
  if (b > sms * 8) b = sms * 8;
  return static_cast<int>(b < 1 ? 1 : b);
}

}  // namespace

int64_t gram_blocks(int64_t rows) { return (rows + kRowsPerBlock - 1) / kRowsPerBlock; }

void launch_gram(const float* partial, int splits, int64_t rows, int lp, float* Y, double* gpart, double* G,
                 cudaStream_t s) {
  const int nb = static_cast<int>(gram_blocks(rows));
  gram_kernel<<<nb, 256, kRowsPerBlock * (lp + 1) * sizeof(float), s>>>(partial, splits, rows, lp, Y, gpart);
  launch_gram_reduce(gpart, nb, lp, G, s);
}

void launch_gram_reduce(const double* gpart, int nblocks, int lp, double* G, cudaStream_t s) {
  const int n2 = lp * lp;
  gram_reduce_kernel<<<(n2 + 255) / 256, 256, 0, s>>>(gpart, nblocks, n2, G);
}

void launch_cholesky_inv(const double* G, int lp, float* Rinv, cudaStream_t s) {
  const size_t smem = (2 * static_cast<size_t>(lp) * (lp + 1) + 2 * lp) * sizeof(double);
  if (!ensure_smem(reinterpret_cast<const void*>(cholesky_inv_kernel), smem)) return;
  cholesky_inv_kernel<<<1, 512, smem, s>>>(G, lp, Rinv);
}

void launch_apply(const ApplyArgs& a, cudaStream_t s) {
  const size_t smem = (static_cast<size_t>(a.kin) * a.kout + kRowsPerBlock * (a.kin + 1) +
                       kRowsPerBlock * (a.kout + 1)) * sizeof(float);
  if (!ensure_smem(reinterpret_cast<const void*>(apply_kernel), smem)) return;
  apply_kernel<<<static_cast<unsigned>(gram_blocks(a.rows)), 256, smem, s>>>(a);
}

void launch_jacobi(const double* C, int n, int max_sweeps, double* eval, float* evec, int32_t* dev_status,
                   cudaStream_t s) {
  const int threads = 512;
  const size_t smem = (2 * static_cast<size_t>(n) * (n + 1) + n + threads) * sizeof(double);
  if (!ensure_smem(reinterpret_cast<const void*>(jacobi_kernel), smem)) return;
  jacobi_kernel<<<1, threads, smem, s>>>(C, n, max_sweeps, 1e-13, eval, evec, dev_status);
}

void launch_factor_mats(const double* eval, const float* evec, int lp, int k, float* Mu, float* Mv, float* S,
                        cudaStream_t s) {
  factor_mats_kernel<<<1, 256, 0, s>>>(eval, evec, lp, k, Mu, Mv, S);
}

int64_t sign_blocks(int64_t rows) { return (rows + 255) / 256; }

void launch_signs(float* U, int64_t m, float* V, int64_t n, int k, float* bmax, int64_t* bidx, float* sign, int sms,
                  cudaStream_t s) {
  const int nb = static_cast<int>(sign_blocks(m));
  colmax_kernel<<<nb, 128, 0, s>>>(U, m, k, bmax, bidx);
  sign_kernel<<<1, 128, 0, s>>>(U, bmax, bidx, nb, k, sign);
  flip_kernel<<<blocks(m * k, sms), 256, 0, s>>>(U, m, k, sign);
  flip_kernel<<<blocks(n * k, sms), 256, 0, s>>>(V, n, k, sign);
}

}  // namespace metis
