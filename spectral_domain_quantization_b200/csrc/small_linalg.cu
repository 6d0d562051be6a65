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
// row stride ld, cols a multiple of 4): out[i][j] for all i, j (symmetric).
// Each thread accumulates a 4 x 4 tile (16 independent float64 chains).
MDEV void gram_block(const float* ys, int rows, int cols, int ld, double* out) {
  const int nb = cols / 4;
  const int npairs = nb * (nb + 1) / 2;
  for (int pidx = threadIdx.x; pidx < npairs; pidx += blockDim.x) {
    int bi = 0, rem = pidx;
    while (rem >= nb - bi) {
      rem -= nb - bi;
      ++bi;
    }
    const int bj = bi + rem;
    double acc[4][4];
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int y = 0; y < 4; ++y) acc[x][y] = 0.0;
    for (int r = 0; r < rows; ++r) {
      const float* row = ys + r * ld;
      double a[4], b[4];
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        a[x] = row[4 * bi + x];
        b[x] = row[4 * bj + x];
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = fma(a[x], b[y], acc[x][y]);
    }
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int y = 0; y < 4; ++y) {
        out[(4 * bi + x) * cols + 4 * bj + y] = acc[x][y];
        out[(4 * bj + y) * cols + 4 * bi + x] = acc[x][y];
      }
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

// One warp per Gram entry: lanes take blocks lane, lane+32, ... and the warp
// reduces with a fixed shuffle tree (deterministic).
__global__ void gram_reduce_kernel(const double* gpart, int nblocks, int n2, double* G) {
  const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (e >= n2) return;
  double s = 0.0;
  for (int b = lane; b < nblocks; b += 32) s += gpart[static_cast<int64_t>(b) * n2 + e];
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  if (lane == 0) G[e] = s;
}

// Decode e -> (q, e - q*d) for e < 2^22 with a float reciprocal (exact).
MDEV int fdiv_index(int e, float rcp) { return __float2int_rz((static_cast<float>(e) + 0.5f) * rcp); }

// G = L L^T (with drops), then Rinv = L^-T (upper triangular, float32).
// Work is enumerated over flattened index ranges so every thread gets an equal
// share of the shrinking triangle.  One barrier per column: step j updates the
// trailing lower triangle with the unscaled column j (times 1/d_j) and scales
// column j-1; the thread updating the next diagonal entry computes the next
// pivot's reciprocal square root, overlapping its latency with the update.
__global__ void __launch_bounds__(1024) cholesky_inv_kernel(const double* G, int lp, float* Rinv) {
  extern __shared__ double sm[];
  const int ld = lp + 1;
  double* L = sm;                  // lp x ld
  double* X = L + lp * ld;         // lp x ld, becomes L^-1
  double* diag0 = X + lp * ld;     // lp
  double* invd = diag0 + lp;       // lp: 1/sqrt(pivot) (0 when dropped)
  double* sqd = invd + lp;         // lp: sqrt(pivot) (0 when dropped)
  const int t = threadIdx.x, nt = blockDim.x;
  for (int e = t; e < lp * lp; e += nt) {
    const int i = e / lp, j = e - i * lp;
    L[i * ld + j] = G[e];
    X[i * ld + j] = i == j ? 1.0 : 0.0;
  }
  for (int i = t; i < lp; i += nt) diag0[i] = G[i * lp + i];
  __syncthreads();
  if (t == 0) {
    const double d = L[0];
    const bool drop = !(diag0[0] > 0.0) || !(d > kDropTol * diag0[0]);
    sqd[0] = drop ? 0.0 : sqrt(d);
    invd[0] = drop ? 0.0 : 1.0 / sqd[0];
  }
  __syncthreads();
  for (int j = 0; j < lp; ++j) {
    const double inv2 = invd[j] * invd[j];
    // trailing lower triangle {(i, c): j < c <= i < lp}, row by row:
    // row i = j + 1 + a holds a + 1 entries; flatten with a triangular decode
    const int w = lp - j - 1;
    const int total = w * (w + 1) / 2;
    for (int e = t; e < total; e += nt) {
      int a = static_cast<int>((sqrtf(8.f * e + 1.f) - 1.f) * 0.5f);
      if ((a + 1) * (a + 2) / 2 <= e) ++a;
      if (a * (a + 1) / 2 > e) --a;
      const int i = j + 1 + a, c = j + 1 + (e - a * (a + 1) / 2);
      const double v = L[i * ld + c] - L[i * ld + j] * L[c * ld + j] * inv2;
      L[i * ld + c] = v;
      if (e == 0) {  // (j+1, j+1): next pivot
        const bool drop = !(diag0[c] > 0.0) || !(v > kDropTol * diag0[c]);
        const double r = drop ? 0.0 : sqrt(v);
        sqd[c] = r;
        invd[c] = drop ? 0.0 : 1.0 / r;
      }
    }
    if (j > 0) {  // deferred scaling of column j-1
      const double pinv = invd[j - 1];
      for (int i = j + t; i < lp; i += nt) L[i * ld + j - 1] *= pinv;
      if (t == 0) L[(j - 1) * ld + j - 1] = sqd[j - 1];
    }
    __syncthreads();
  }
  if (t == 0) L[(lp - 1) * ld + lp - 1] = sqd[lp - 1];
  // X = L^-1: step k eliminates with the unscaled row k (times 1/L_kk) over
  // the rectangle rows k+1.., columns 0..k, and scales row k-1
  for (int k = 0; k < lp; ++k) {
    const double inv = invd[k];
    const int cols = k + 1, total = (lp - k - 1) * cols;
    const float rcp = 1.f / static_cast<float>(cols);
    for (int e = t; e < total; e += nt) {
      const int q = fdiv_index(e, rcp);
      const int i = k + 1 + q, c = e - q * cols;
      X[i * ld + c] -= L[i * ld + k] * inv * X[k * ld + c];
    }
    if (k > 0) {
      const double pinv = invd[k - 1];
      for (int c = t; c < k; c += nt) X[(k - 1) * ld + c] *= pinv;
    }
    __syncthreads();
  }
  for (int c = t; c < lp; c += nt) X[(lp - 1) * ld + c] *= invd[lp - 1];
  __syncthreads();
  for (int e = t; e < lp * lp; e += nt) {
    const int j = e / lp, c = e - j * lp;  // Rinv[j][c] = X[c][j]
    Rinv[e] = c >= j ? static_cast<float>(X[c * ld + j]) : 0.f;
  }
}

constexpr int kApplyRows = 32;

// out = in (rows x kin) * M (kin x kout).  32 rows per CTA, 256 threads, each
// thread a 2-row x ceil(kout/16)-column register tile.  Optional fp32 out,
// transposed bf16 hi/lo copy, Gram partial of the output block.
__global__ void __launch_bounds__(256) apply_kernel(ApplyArgs a) {
  extern __shared__ float smf[];
  float* Ms = smf;                                   // kin x kout
  float* In = Ms + a.kin * a.kout;                   // kApplyRows x (kin + 1)
  float* Out = In + kApplyRows * (a.kin + 1);        // kApplyRows x (kout + 1)
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kApplyRows;
  const int nr = static_cast<int>(imin64(kApplyRows, a.rows - r0));
  for (int e = threadIdx.x; e < a.kin * a.kout; e += blockDim.x) Ms[e] = a.M[e];
  for (int e = threadIdx.x; e < kApplyRows * a.kin; e += blockDim.x) {
    const int r = e / a.kin, c = e - r * a.kin;
    In[r * (a.kin + 1) + c] = r < nr ? a.in[(r0 + r) * a.in_ld + c] : 0.f;
  }
  __syncthreads();
  const int tr = threadIdx.x & 15, tc = threadIdx.x >> 4;
  constexpr int kMaxCols = 7;  // kout <= 112
  float acc[2][kMaxCols];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int u = 0; u < kMaxCols; ++u) acc[i][u] = 0.f;
  const float* in0 = In + (2 * tr) * (a.kin + 1);
  const float* in1 = in0 + (a.kin + 1);
#pragma unroll 2
  for (int j = 0; j < a.kin; ++j) {
    const float x0 = in0[j], x1 = in1[j];
    const float* mrow = Ms + j * a.kout;
#pragma unroll
    for (int u = 0; u < kMaxCols; ++u) {
      const int c = tc + 16 * u;
      const float m = c < a.kout ? mrow[c] : 0.f;
      acc[0][u] = fmaf(x0, m, acc[0][u]);
      acc[1][u] = fmaf(x1, m, acc[1][u]);
    }
  }
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int u = 0; u < kMaxCols; ++u) {
      const int c = tc + 16 * u;
      if (c < a.kout) Out[(2 * tr + i) * (a.kout + 1) + c] = acc[i][u];
    }
  __syncthreads();
  for (int e = threadIdx.x; e < kApplyRows * a.kout; e += blockDim.x) {
    if (a.out) {
      const int r = e / a.kout, c = e - r * a.kout;  // column fastest: coalesced rows
      if (r < nr) a.out[(r0 + r) * a.out_ld + c] = Out[r * (a.kout + 1) + c];
    }
    if (a.outT) {
      const int c = e / kApplyRows, r = e - c * kApplyRows;  // row fastest: coalesced columns of out^T
      if (r < nr) {
        const float v = Out[r * (a.kout + 1) + c];
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        a.outT[static_cast<int64_t>(c) * a.ldx + r0 + r] = hi;
        a.outT[static_cast<int64_t>(a.lpT + c) * a.ldx + r0 + r] = __float2bfloat16_rn(__fsub_rn(v, __bfloat162float(hi)));
      }
    }
  }
  if (a.gpart) gram_block(Out, nr, a.kout, a.kout + 1, a.gpart + static_cast<int64_t>(blockIdx.x) * a.kout * a.kout);
}

// Round-robin pairing: in step r of a sweep over n (even) indices, slot i
// pairs with slot n-1-i; slot 0 holds index 0, slots 1..n-1 rotate.
MDEV int rr_index(int slot, int step, int n) {
  if (slot == 0) return 0;
  return ((slot - 1 + step) % (n - 1)) + 1;
}

constexpr double kRankTol = 1e-10;   // pivoted Cholesky: relative diagonal cut
// one-sided Jacobi: rotate while |a.b| > tol |a||b|.  Float32 sums of <= 112
// products carry ~5e-7 relative noise, so the rule sits well above it.
constexpr float kJacobiTol = 4e-6f;

// Eigen-decomposition of the l x l core Gram C = Z^T Z (PSD), eigenvalues
// descending; evec[i * n + j] = component i of eigenvector j.
//   1. pivoted Cholesky (float64): P C P^T = L L^T (rank-revealing cut);
//   2. one-sided Jacobi on the columns of L (float32, eight lanes per column
//      pair, round-robin order): L J = U diag(sigma), so the normalised
//      columns are the eigenvectors of P C P^T and sigma^2 its eigenvalues
//      (this is the one-sided Jacobi SVD of the core, preconditioned by the
//      pivoted factorization, which needs few sweeps);
//   3. sort and undo the pivoting.
__global__ void __launch_bounds__(1024) core_eig_kernel(const double* C, int n, int max_sweeps, double* eval,
                                                        float* evec, int32_t* dev_status) {
  extern __shared__ double smd[];
  const int ld = n + 1;
  double* G = smd;                                       // n x ld
  float* X = reinterpret_cast<float*>(G + n * ld);       // column j at X[j * ld + r]
  int* perm = reinterpret_cast<int*>(X + n * ld);        // n
  float* norms = reinterpret_cast<float*>(perm + n);     // n
  __shared__ int piv_sh, rotated_sh;
  __shared__ double maxd_sh;
  const int t = threadIdx.x, nt = blockDim.x, warp = t >> 5, lane = t & 31, nwarps = nt >> 5;
  for (int e = t; e < n * n; e += nt) G[(e / n) * ld + e % n] = C[e];
  for (int i = t; i < n; i += nt) perm[i] = i;
  __syncthreads();
  if (warp == 0) {
    double m = 0.0;
    for (int i = lane; i < n; i += 32) m = fmax(m, G[i * ld + i]);
    for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (lane == 0) maxd_sh = m;
  }
  __syncthreads();
  const double cut = kRankTol * maxd_sh;
  int rank = n;
  for (int j = 0; j < n; ++j) {
    if (warp == 0) {
      double best = -1.0;
      int bi = j;
      for (int i = j + lane; i < n; i += 32) {
        const double v = G[i * ld + i];
        if (v > best) {
          best = v;
          bi = i;
        }
      }
      for (int o = 16; o > 0; o >>= 1) {
        const double ob = __shfl_xor_sync(0xFFFFFFFFu, best, o);
        const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
        if (ob > best || (ob == best && oi < bi)) {
          best = ob;
          bi = oi;
        }
      }
      if (lane == 0) piv_sh = bi;
    }
    __syncthreads();
    const int p = piv_sh;
    if (p != j) {
      for (int c = t; c < n; c += nt) {
        const double a = G[j * ld + c];
        G[j * ld + c] = G[p * ld + c];
        G[p * ld + c] = a;
      }
      __syncthreads();
      for (int r = t; r < n; r += nt) {
        const double a = G[r * ld + j];
        G[r * ld + j] = G[r * ld + p];
        G[r * ld + p] = a;
      }
      if (t == 0) {
        const int a = perm[j];
        perm[j] = perm[p];
        perm[p] = a;
      }
      __syncthreads();
    }
    const double d = G[j * ld + j];
    if (!(d > cut)) {
      rank = j;
      break;
    }
    const double inv = 1.0 / sqrt(d);
    const double invd2 = inv * inv;
    // the whole (symmetric) Schur complement is kept current, so that the
    // next pivot swap can exchange complete rows and columns
    const int w = n - j - 1;
    const float rcpw = 1.f / static_cast<float>(w > 0 ? w : 1);
    for (int e = t; e < w * w; e += nt) {
      const int q = fdiv_index(e, rcpw);
      const int i = j + 1 + q, c = j + 1 + (e - q * w);
      G[i * ld + c] -= G[i * ld + j] * G[c * ld + j] * invd2;
    }
    __syncthreads();
    for (int i = j + 1 + t; i < n; i += nt) G[i * ld + j] *= inv;
    if (t == 0) G[j * ld + j] = d * inv;
    __syncthreads();
  }
  for (int e = t; e < n * n; e += nt) {
    const int j = e / n, r = e - j * n;
    X[j * ld + r] = (j < rank && r >= j) ? static_cast<float>(G[r * ld + j]) : 0.f;
  }
  __syncthreads();
  // one-sided Jacobi: 8 lanes per column pair, 4 pairs per warp
  const int grp = lane >> 3, l8 = lane & 7;
  const int npairs = n / 2;
  int sweep = 0;
  for (; sweep < max_sweeps; ++sweep) {
    if (t == 0) rotated_sh = 0;
    __syncthreads();
    for (int step = 0; step < n - 1; ++step) {
      for (int base = 4 * warp; base < npairs; base += 4 * nwarps) {
        const int pair = base + grp;
        const bool act = pair < npairs;
        int p = 0, q = 1;
        if (act) {
          p = rr_index(pair, step, n);
          q = rr_index(n - 1 - pair, step, n);
          if (p > q) {
            const int x = p;
            p = q;
            q = x;
          }
        }
        float al = 0.f, be = 0.f, ga = 0.f;
        if (act) {
          for (int r = l8; r < n; r += 8) {
            const float a = X[p * ld + r], b = X[q * ld + r];
            al = fmaf(a, a, al);
            be = fmaf(b, b, be);
            ga = fmaf(a, b, ga);
          }
        }
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) {
          al += __shfl_xor_sync(0xFFFFFFFFu, al, o);
          be += __shfl_xor_sync(0xFFFFFFFFu, be, o);
          ga += __shfl_xor_sync(0xFFFFFFFFu, ga, o);
        }
        if (act && ga != 0.f && fabsf(ga) > kJacobiTol * sqrtf(al * be)) {
          const float zeta = (be - al) / (2.f * ga);
          const float tt = copysignf(1.f, zeta) / (fabsf(zeta) + sqrtf(fmaf(zeta, zeta, 1.f)));
          const float c = rsqrtf(fmaf(tt, tt, 1.f));
          const float s = c * tt;
          for (int r = l8; r < n; r += 8) {
            const float a = X[p * ld + r], b = X[q * ld + r];
            X[p * ld + r] = c * a - s * b;
            X[q * ld + r] = s * a + c * b;
          }
          if (l8 == 0) rotated_sh = 1;
        }
      }
      __syncthreads();
    }
    if (!rotated_sh) break;
  }
  if (t == 0 && sweep >= max_sweeps) report(dev_status, METIS_DEV_NUMERIC);
  for (int j = t; j < n; j += nt) {
    double s2 = 0.0;
    for (int r = 0; r < n; ++r) s2 += static_cast<double>(X[j * ld + r]) * X[j * ld + r];
    norms[j] = static_cast<float>(sqrt(s2));
  }
  __syncthreads();
  for (int j = t; j < n; j += nt) {
    const float sj = norms[j];
    int rk = 0;
    for (int i = 0; i < n; ++i) {
      const float si = norms[i];
      rk += (si > sj) || (si == sj && i < j);
    }
    eval[rk] = static_cast<double>(sj) * sj;
    const float inv = sj > 0.f ? 1.f / sj : 0.f;
    for (int r = 0; r < n; ++r) evec[perm[r] * n + rk] = X[j * ld + r] * inv;
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

int64_t apply_blocks(int64_t rows) { return (rows + kApplyRows - 1) / kApplyRows; }

void launch_gram(const float* partial, int splits, int64_t rows, int lp, float* Y, double* gpart, double* G,
                 cudaStream_t s) {
  const int nb = static_cast<int>(gram_blocks(rows));
  gram_kernel<<<nb, 256, kRowsPerBlock * (lp + 1) * sizeof(float), s>>>(partial, splits, rows, lp, Y, gpart);
  launch_gram_reduce(gpart, nb, lp, G, s);
}

void launch_gram_reduce(const double* gpart, int nblocks, int lp, double* G, cudaStream_t s) {
  const int n2 = lp * lp;
  gram_reduce_kernel<<<(n2 + 7) / 8, 256, 0, s>>>(gpart, nblocks, n2, G);
}

void launch_cholesky_inv(const double* G, int lp, float* Rinv, cudaStream_t s) {
  const size_t smem = (2 * static_cast<size_t>(lp) * (lp + 1) + 3 * lp) * sizeof(double);
  if (!ensure_smem(reinterpret_cast<const void*>(cholesky_inv_kernel), smem)) return;
  cholesky_inv_kernel<<<1, 1024, smem, s>>>(G, lp, Rinv);
}

void launch_apply(const ApplyArgs& a, cudaStream_t s) {
  const size_t smem = (static_cast<size_t>(a.kin) * a.kout + kApplyRows * (a.kin + 1) +
                       kApplyRows * (a.kout + 1)) * sizeof(float);
  if (!ensure_smem(reinterpret_cast<const void*>(apply_kernel), smem)) return;
  apply_kernel<<<static_cast<unsigned>(apply_blocks(a.rows)), 256, smem, s>>>(a);
}

void launch_jacobi(const double* C, int n, int max_sweeps, double* eval, float* evec, int32_t* dev_status,
                   cudaStream_t s) {
  const size_t smem = static_cast<size_t>(n) * (n + 1) * sizeof(double) + static_cast<size_t>(n) * (n + 1) * sizeof(float) +
                      2 * static_cast<size_t>(n) * sizeof(int);
  if (!ensure_smem(reinterpret_cast<const void*>(core_eig_kernel), smem)) return;
  core_eig_kernel<<<1, 1024, smem, s>>>(C, n, max_sweeps, eval, evec, dev_status);
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
