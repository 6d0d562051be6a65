// Symmetric eigen-decomposition of the small core Gram C = Z^T Z (n <= 112,
// float64): the "small core SVD" step of the randomized split.
//
// Source: SII release on Metis, section 2.4 item 1 (the decomposition of the
// low-dimensional sketch separates the dominant directions from the long
// tail); "Metis: Training LLMs with FP4 Quantization" technical framework
// (random projection followed by a small decomposition).  C's eigenvectors W
// and eigenvalues sigma^2 give the core SVD: U = Q W, V = Z W / sigma.
//
// The problem is tiny and latency-bound, so the work is cut into three
// launches that each keep their sequential chains short:
//   1. core_tridiag_kernel (one CTA): Householder reduction C = Q T Q^T to a
//      symmetric tridiagonal T (diagonal d, off-diagonal e), accumulating Q;
//      three barriers per column.
//   2. core_vector_kernel (one CTA of one warp per eigenvalue): the
//      eigenvalue by multisection on Sturm counts (32 points per round, the
//      counts from the division-free determinant recurrence with power-of-two
//      rescaling), then its eigenvector from the twisted factorization of
//      T - lambda I (the twist at the smallest |gamma_r|), normalised and
//      taken back through Q.
//   3. core_finish_kernel (one CTA): re-orthogonalises the vectors of
//      eigenvalue clusters (modified Gram-Schmidt, with an orthogonal
//      completion for a vector that collapses, as in an exactly degenerate
//      cluster), then writes eigenvalues in descending order and the float32
//      eigenvectors in the same order.
#include "abi_common.h"
#include "common.cuh"
#include "small_linalg.h"

namespace metis {

namespace {

constexpr int kTriThreads = 1024;
constexpr int kMaxN = 112;
constexpr double kClusterTol = 1e-9; // relative gap below which vectors are re-orthogonalised

// Scratch layout (doubles): Q [n][n], X [n][n] (eigenvectors, column idx =
// eigenvalue idx in ascending order), d [n], e [n], lam [n].
struct EigScratch {
  double *Q, *X, *d, *e, *lam;
};

__host__ __device__ inline EigScratch scratch(double* ws, int n) {
  EigScratch s;
  s.Q = ws;
  s.X = s.Q + n * n;
  s.d = s.X + n * n;
  s.e = s.d + n;
  s.lam = s.e + n;
  return s;
}

// ---------------------------------------------------------------------------
// 1. Householder tridiagonalisation
// ---------------------------------------------------------------------------
// Column j: x = A[j+1.., j], alpha = -sign(x0) |x|, v = x - alpha e_1,
// beta = 2 / v^T v, p = beta A' v, w = p - (beta/2)(p^T v) v,
// A' -= v w^T + w v^T, Q[:, j+1..] -= beta (Q[:, j+1..] v) v^T.
__global__ void __launch_bounds__(kTriThreads) core_tridiag_kernel(const double* C, int n, double* ws) {
  extern __shared__ double sm[];
  const int ld = n + 1;
  double* A = sm;             // n x ld
  double* Qs = A + n * ld;    // n x ld
  double* vb = Qs + n * ld;   // n: Householder vector
  double* pb = vb + n;        // n: beta A' v
  double* qb = pb + n;        // n: Q' v
  const EigScratch S = scratch(ws, n);
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  constexpr int kWarps = kTriThreads / 32;
  for (int e = t; e < n * n; e += kTriThreads) {
    const int i = e / n, c = e - i * n;
    A[i * ld + c] = C[e];
    Qs[i * ld + c] = i == c ? 1.0 : 0.0;
  }
  __syncthreads();
  for (int j = 0; j + 2 < n; ++j) {
    const int m = n - j - 1;  // rows / columns j+1 .. n-1
    // every warp: the norm of x below its first entry (same order: same value)
    double sg = 0.0;
    for (int i = 1 + lane; i < m; i += 32) {
      const double x = A[(j + 1 + i) * ld + j];
      sg = fma(x, x, sg);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sg += __shfl_xor_sync(0xFFFFFFFFu, sg, o);
    const double x0 = A[(j + 1) * ld + j];
    double alpha = x0, beta = 0.0, v0 = 0.0;
    if (sg > 0.0) {
      const double nrm = sqrt(fma(x0, x0, sg));
      alpha = x0 >= 0.0 ? -nrm : nrm;
      v0 = x0 - alpha;
      beta = 2.0 / fma(v0, v0, sg);
    }
    if (t == 0) {
      S.d[j] = A[j * ld + j];
      S.e[j] = alpha;
    }
    if (beta != 0.0) {  // uniform: every thread computed the same sg
      for (int i = t; i < m; i += kTriThreads) vb[i] = i == 0 ? v0 : A[(j + 1 + i) * ld + j];
      __syncthreads();
      // p (rows 0..m-1 of A') and q (rows 0..n-1 of Q'): eight lanes per row
      const int g = lane >> 3, l8 = lane & 7;
      for (int base = 4 * warp; base < m + n; base += 4 * kWarps) {
        const int row = base + g;
        double s = 0.0;
        if (row < m) {
          const double* ar = A + (j + 1 + row) * ld + j + 1;
          for (int k = l8; k < m; k += 8) s = fma(ar[k], vb[k], s);
        } else if (row < m + n) {
          const double* qr = Qs + (row - m) * ld + j + 1;
          for (int k = l8; k < m; k += 8) s = fma(qr[k], vb[k], s);
        }
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
        if (l8 == 0) {
          if (row < m) pb[row] = beta * s;
          else if (row < m + n) qb[row - m] = s;
        }
      }
      __syncthreads();
      // K = (beta / 2) p^T v, every warp
      double kk = 0.0;
      for (int i = lane; i < m; i += 32) kk = fma(pb[i], vb[i], kk);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) kk += __shfl_xor_sync(0xFFFFFFFFu, kk, o);
      const double K = 0.5 * beta * kk;
      // A' -= v w^T + w v^T: warp rows, lane columns
      for (int i = warp; i < m; i += kWarps) {
        const double vi = vb[i], wi = pb[i] - K * vi;
        double* ar = A + (j + 1 + i) * ld + j + 1;
        for (int k = lane; k < m; k += 32) {
          const double vk = vb[k], wk = pb[k] - K * vk;
          ar[k] -= fma(vi, wk, wi * vk);
        }
      }
      // Q' -= beta q v^T
      for (int r = warp; r < n; r += kWarps) {
        const double qr = beta * qb[r];
        double* q = Qs + r * ld + j + 1;
        for (int k = lane; k < m; k += 32) q[k] -= qr * vb[k];
      }
    }
    __syncthreads();
  }
  if (t == 0) {
    S.d[n - 2] = A[(n - 2) * ld + n - 2];
    S.d[n - 1] = A[(n - 1) * ld + n - 1];
    S.e[n - 2] = A[(n - 1) * ld + n - 2];
  }
  for (int e = t; e < n * n; e += kTriThreads) {
    const int i = e / n, c = e - i * n;
    S.Q[e] = Qs[i * ld + c];
  }
}

// ---------------------------------------------------------------------------
// 2. one eigenpair per CTA (one warp)
// ---------------------------------------------------------------------------

// Number of eigenvalues of T below x (scaled T: |d|, |e| <= 1): sign changes
// of the leading principal minors p_{-1} = 1, p_0, ..., p_{n-1}, with
// p_i = (d_i - x) p_{i-1} - e_{i-1}^2 p_{i-2}; a zero minor takes the sign of
// the one before it.  The pair (p_{i-1}, p_i) is rescaled by a power of two
// every fourth step (|p| grows at most 5x per step), so nothing overflows.
MDEV int sturm_count(const double* d, const double* e2, int n, double x) {
  double pm2 = 1.0, pm1 = d[0] - x;
  int sg = 1, cnt = 0;
  {
    const int s = pm1 < 0.0 ? -1 : (pm1 > 0.0 ? 1 : sg);
    cnt += s != sg;
    sg = s;
  }
  for (int i = 1; i < n; ++i) {
    const double p = fma(d[i] - x, pm1, -e2[i - 1] * pm2);
    const int s = p < 0.0 ? -1 : (p > 0.0 ? 1 : sg);
    cnt += s != sg;
    sg = s;
    pm2 = pm1;
    pm1 = p;
    if ((i & 3) == 0) {
      const double ref = fmax(fabs(pm1), fabs(pm2));
      if (ref != 0.0) {
        const int ex = ilogb(ref);
        pm1 = ldexp(pm1, -ex);
        pm2 = ldexp(pm2, -ex);
      }
    }
  }
  return cnt;
}

__global__ void __launch_bounds__(32) core_vector_kernel(int n, double* ws, int max_rounds, int32_t* dev_status) {
  __shared__ double d[kMaxN], e[kMaxN], e2[kMaxN], dp[kMaxN], lp[kMaxN], um[kMaxN], z[kMaxN];
  const EigScratch S = scratch(ws, n);
  const int lane = threadIdx.x, idx = blockIdx.x;  // eigenvalue idx in ascending order
  // scale T by a power of two so that |d|, |e| <= 1
  double mx = 0.0;
  for (int i = lane; i < n; i += 32) {
    mx = fmax(mx, fabs(S.d[i]));
    if (i + 1 < n) mx = fmax(mx, fabs(S.e[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  if (mx == 0.0) {  // T = 0: every unit vector is an eigenvector
    for (int r = lane; r < n; r += 32) S.X[r * n + idx] = S.Q[r * n + idx];
    if (lane == 0) S.lam[idx] = 0.0;
    return;
  }
  int ex;
  frexp(mx, &ex);  // mx < 2^ex
  for (int i = lane; i < n; i += 32) {
    d[i] = ldexp(S.d[i], -ex);
    const double ei = i + 1 < n ? ldexp(S.e[i], -ex) : 0.0;
    e[i] = ei;
    e2[i] = ei * ei;
  }
  __syncwarp();
  // Gershgorin interval
  double lo = 1e300, hi = -1e300;
  for (int i = lane; i < n; i += 32) {
    const double r = fabs(e[i]) + (i > 0 ? fabs(e[i - 1]) : 0.0);
    lo = fmin(lo, d[i] - r);
    hi = fmax(hi, d[i] + r);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fmin(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
    hi = fmax(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
  }
  lo -= 1e-12;
  hi += 1e-12;
  // multisection: the smallest x with count(x) > idx
  bool done = false;
  for (int round = 0; round < max_rounds; ++round) {
    if (hi - lo <= 0x1p-50 * fmax(fabs(lo), fabs(hi)) + 0x1p-60) {
      done = true;
      break;
    }
    const double x = lo + (hi - lo) * (static_cast<double>(lane + 1) / 33.0);
    const int c = sturm_count(d, e2, n, x);
    const unsigned mask = __ballot_sync(0xFFFFFFFFu, c > idx);
    const double x_prev = __shfl_up_sync(0xFFFFFFFFu, x, 1);
    if (mask) {
      const int f = __ffs(mask) - 1;
      const double nlo = f > 0 ? __shfl_sync(0xFFFFFFFFu, x_prev, f) : lo;
      hi = __shfl_sync(0xFFFFFFFFu, x, f);
      lo = nlo;
    } else {
      lo = __shfl_sync(0xFFFFFFFFu, x, 31);
    }
  }
  if (!done && lane == 0) report(dev_status, METIS_DEV_NUMERIC);
  const double lam = 0.5 * (lo + hi);
  // twisted factorisation of T - lam I (lane 0; the recurrences are serial)
  if (lane == 0) {
    const double pivmin = 0x1p-100;
    double Dp = d[0] - lam;
    for (int i = 0; i + 1 < n; ++i) {
      if (fabs(Dp) < pivmin) Dp = Dp < 0.0 ? -pivmin : pivmin;
      dp[i] = Dp;
      lp[i] = e[i] / Dp;
      Dp = (d[i + 1] - lam) - lp[i] * e[i];
    }
    dp[n - 1] = Dp;
    double Dm = d[n - 1] - lam;
    int r = n - 1;
    double best = fabs(dp[n - 1]);  // gamma_{n-1} = D+_{n-1}
    for (int i = n - 1; i > 0; --i) {
      if (fabs(Dm) < pivmin) Dm = Dm < 0.0 ? -pivmin : pivmin;
      um[i - 1] = e[i - 1] / Dm;
      const double a = d[i - 1] - lam;
      Dm = a - um[i - 1] * e[i - 1];
      const double g = fabs(dp[i - 1] + Dm - a);
      if (g < best) {
        best = g;
        r = i - 1;
      }
    }
    z[r] = 1.0;
    for (int i = r - 1; i >= 0; --i) {
      z[i] = -lp[i] * z[i + 1];
      if (fabs(z[i]) > 1e150)
        for (int q = i; q <= r; ++q) z[q] *= 1e-150;
    }
    for (int i = r; i + 1 < n; ++i) {
      z[i + 1] = -um[i] * z[i];
      if (fabs(z[i + 1]) > 1e150)
        for (int q = 0; q <= i + 1; ++q) z[q] *= 1e-150;
    }
  }
  __syncwarp();
  double nrm = 0.0;
  for (int i = lane; i < n; i += 32) nrm = fma(z[i], z[i], nrm);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) nrm += __shfl_xor_sync(0xFFFFFFFFu, nrm, o);
  const double inv = 1.0 / sqrt(nrm);
  // back to the basis of C: x = Q z
  for (int r = lane; r < n; r += 32) {
    const double* q = S.Q + r * n;
    double s = 0.0;
    for (int k = 0; k < n; ++k) s = fma(q[k], z[k], s);
    S.X[r * n + idx] = s * inv;
  }
  if (lane == 0) S.lam[idx] = ldexp(lam, ex);
}

// ---------------------------------------------------------------------------
// 3. clusters, order, float32 output
// ---------------------------------------------------------------------------

// v -= (x_s . v) x_s for every column s of X with use(s) (one warp; column
// entries r = lane + 32 q held in v[q]).
template <typename Use>
MDEV void project_out(const double* X, int n, double* v, Use use) {
  const int lane = threadIdx.x & 31;
  for (int s = 0; s < n; ++s) {
    if (!use(s)) continue;
    double c = 0.0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = lane + 32 * q;
      if (r < n) c = fma(X[r * n + s], v[q], c);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = lane + 32 * q;
      if (r < n) v[q] = fma(-c, X[r * n + s], v[q]);
    }
  }
}

MDEV double warp_norm(const double* v, int n) {
  const int lane = threadIdx.x & 31;
  double s = 0.0;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (lane + 32 * q < n) s = fma(v[q], v[q], s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  return sqrt(s);
}

__global__ void __launch_bounds__(256) core_finish_kernel(int n, double* ws, double* eval, float* evec) {
  const EigScratch S = scratch(ws, n);
  double* X = S.X;
  if (threadIdx.x < 32) {
    double top = 0.0;
    for (int i = 0; i < n; ++i) top = fmax(top, fabs(S.lam[i]));
    const double tol = kClusterTol * top;
    int c0 = 0, cand = 0;
    while (c0 < n) {
      int c1 = c0 + 1;  // cluster [c0, c1)
      while (c1 < n && S.lam[c1] - S.lam[c1 - 1] <= tol) ++c1;
      for (int t = c0 + 1; t < c1; ++t) {
        double v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int r = threadIdx.x + 32 * q;
          v[q] = r < n ? X[r * n + t] : 0.0;
        }
        auto earlier = [&](int s) { return s >= c0 && s < t; };
        project_out(X, n, v, earlier);
        project_out(X, n, v, earlier);
        double nv = warp_norm(v, n);
        if (nv < 0.5) {
          // collapsed: complete with a unit vector projected off every other
          // column already fixed (all outside [t, c1) )
          // (the unit-vector candidates are tried in order across the whole
          // kernel, so a degenerate cluster costs O(n) candidates in all)
          auto fixed = [&](int s) { return s < t || s >= c1; };
          for (; cand < n; ++cand) {
#pragma unroll
            for (int q = 0; q < 4; ++q) v[q] = threadIdx.x + 32 * q == cand ? 1.0 : 0.0;
            project_out(X, n, v, fixed);
            project_out(X, n, v, fixed);
            nv = warp_norm(v, n);
            if (nv > 0.5) break;
          }
        }
        const double iv = nv > 0.0 ? 1.0 / nv : 0.0;
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int r = threadIdx.x + 32 * q;
          if (r < n) X[r * n + t] = v[q] * iv;
        }
        __syncwarp();
      }
      c0 = c1;
    }
  }
  __syncthreads();
  // descending order: rank = n - 1 - idx
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
    const int r = e / n, rk = e - r * n;
    evec[e] = static_cast<float>(X[r * n + (n - 1 - rk)]);
  }
  for (int i = threadIdx.x; i < n; i += blockDim.x) eval[i] = S.lam[n - 1 - i];
}

}  // namespace

size_t core_eig_workspace(int n) { return (2 * static_cast<size_t>(n) * n + 3 * n) * sizeof(double); }

void launch_core_eig(double* C, int n, int max_iters, double* eval, float* evec, double* ws, int32_t* dev_status,
                     cudaStream_t s) {
  const size_t smem = (2 * static_cast<size_t>(n) * (n + 1) + 3 * n) * sizeof(double);
  if (!ensure_smem(reinterpret_cast<const void*>(core_tridiag_kernel), smem)) return;
  core_tridiag_kernel<<<1, kTriThreads, smem, s>>>(C, n, ws);
  core_vector_kernel<<<n, 32, 0, s>>>(n, ws, max_iters, dev_status);
  core_finish_kernel<<<1, 256, 0, s>>>(n, ws, eval, evec);
}

}  // namespace metis
