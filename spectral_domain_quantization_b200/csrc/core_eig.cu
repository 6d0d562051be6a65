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
//      symmetric tridiagonal T (diagonal d, off-diagonal e), accumulating Q,
//      with A and Q held in per-thread register tiles; three barriers per
//      column.
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

constexpr int kTriThreads = 512;  // >= the 406 tiles of n = 112
constexpr int kMaxN = 112;
constexpr double kClusterTol = 1e-9; // relative gap below which vectors are re-orthogonalised

// Scratch layout (doubles): V [n][n] (Householder vector j in row j, zero
// up to entry j), X [n][n] (eigenvectors, column idx = eigenvalue idx in
// ascending order), d [n], e [n], beta [n], lam [n].
struct EigScratch {
  double *V, *X, *d, *e, *beta, *lam;
};

__host__ __device__ inline EigScratch scratch(double* ws, int n) {
  EigScratch s;
  s.V = ws;
  s.X = s.V + n * n;
  s.d = s.X + n * n;
  s.e = s.d + n;
  s.beta = s.e + n;
  s.lam = s.beta + n;
  return s;
}

// ---------------------------------------------------------------------------
// Tile (I, J), I >= J, of an nb x nb lower block triangle: its index in
// row-major order of the triangle, and the inverse map (packed (I << 8) | J).
MDEV int tri_pos(int I, int J, int) { return I * (I + 1) / 2 + J; }
MDEV int tri_index(int t, int) {
  int I = static_cast<int>((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
  while ((I + 1) * (I + 2) / 2 <= t) ++I;
  while (I * (I + 1) / 2 > t) --I;
  return (I << 8) | (t - I * (I + 1) / 2);
}

// Column c (a runtime index) of a 4 x 4 register tile into dst[0..3],
// selected without dynamic register indexing.
MDEV void publish_col(const double (&a)[4][4], int c, double* dst) {
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    double v = a[r][0];
#pragma unroll
    for (int q = 1; q < 4; ++q) v = q == c ? a[r][q] : v;
    dst[r] = v;
  }
}

// ---------------------------------------------------------------------------
// 1. Householder tridiagonalisation
// ---------------------------------------------------------------------------
// Column j: x = A[j+1.., j], alpha = -sign(x0) |x|, v = x - alpha e_1,
// beta = 2 / v^T v, p = beta A' v, w = p - (beta/2)(p^T v) v,
// A' -= v w^T + w v^T; (v, beta) are kept so that the eigenvectors can be
// taken back through H_0 ... H_{n-3} later.
// Register tiles: thread T < nA owns the 4 x 4 tile (I, J), I >= J, of the
// symmetric A (a diagonal tile holds its whole block).  A step publishes
// nothing but vectors:
//   (a) every tile multiplies by the v it needs (its rows and, off the
//       diagonal, its columns) into per-tile partial sums;
//   (b) one thread per row adds the partials in a fixed order (p);
//   (c) every tile applies its rank-2 update and the tiles holding column
//       j + 1 publish it for the next step.

__global__ void __launch_bounds__(kTriThreads, 1) core_tridiag_kernel(const double* C, int n, double* ws) {
  extern __shared__ double sm[];
  const int nb = n / 4;
  const int nA = nb * (nb + 1) / 2;
  double* xb = sm;                 // 2 x n: column j of A below the diagonal (double-buffered)
  double* pb = xb + 2 * n;         // n: beta A' v
  double* partA = pb + n;          // nA x 4: row sums of each A tile
  double* partT = partA + 4 * nA;  // nA x 4: column sums of each off-diagonal A tile
  const EigScratch S = scratch(ws, n);
  const int t = threadIdx.x, lane = t & 31;
  // ---- tile ownership
  const bool isA = t < nA;
  int I = 0, J = 0;
  double a[4][4];
  if (isA) {
    const int ij = tri_index(t, nb);
    I = ij >> 8;
    J = ij & 255;
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) a[r][c] = C[(4 * I + r) * n + 4 * J + c];
    if (J == 0) {
#pragma unroll
      for (int r = 0; r < 4; ++r) xb[4 * I + r] = a[r][0];
    }
  }
  __syncthreads();
  for (int j = 0; j + 2 < n; ++j) {
    const double* x = xb + (j & 1) * n;        // x[i] = A[i][j], i > j
    double* xn = xb + ((j + 1) & 1) * n;
    // every warp: alpha, beta, v0 (the same arithmetic in every warp)
    double sg = 0.0;
    for (int i = j + 2 + lane; i < n; i += 32) sg = fma(x[i], x[i], sg);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sg += __shfl_xor_sync(0xFFFFFFFFu, sg, o);
    const double x0 = x[j + 1];
    double alpha = x0, beta = 0.0, v0 = 0.0;
    if (sg > 0.0) {
      const double nrm = sqrt(fma(x0, x0, sg));
      alpha = x0 >= 0.0 ? -nrm : nrm;
      v0 = x0 - alpha;
      beta = 2.0 / fma(v0, v0, sg);
    }
    if (t == 0) {
      S.e[j] = alpha;
      S.beta[j] = beta;
    }
    if (isA && I == j / 4 && J == I) {
      const int jm = j % 4;
      double dj = a[0][0];
#pragma unroll
      for (int r = 1; r < 4; ++r) dj = r == jm ? a[r][r] : dj;
      S.d[j] = dj;
    }
    if (beta == 0.0) {  // nothing to eliminate (uniform): column j + 1 is already final
      for (int i = t; i < n; i += kTriThreads) S.V[j * n + i] = 0.0;
      if (isA && J == (j + 1) / 4) publish_col(a, (j + 1) % 4, xn + 4 * I);
      __syncthreads();
      continue;
    }
    auto vel = [&](int i) { return i <= j ? 0.0 : (i == j + 1 ? v0 : x[i]); };
    for (int i = t; i < n; i += kTriThreads) S.V[j * n + i] = vel(i);
    // (a) partial products
    const bool actA = isA && 4 * J + 3 > j;
    if (actA) {
      double vr[4], vc[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        vr[r] = vel(4 * I + r);
        vc[r] = vel(4 * J + r);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        double s = 0.0;
#pragma unroll
        for (int c = 0; c < 4; ++c) s = fma(a[r][c], vc[c], s);
        partA[4 * t + r] = s;
      }
      if (I != J) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          double s = 0.0;
#pragma unroll
          for (int r = 0; r < 4; ++r) s = fma(a[r][c], vr[r], s);
          partT[4 * t + c] = s;
        }
      }
    }
    __syncthreads();
    // (b) p_i (rows i > j): fixed-order sums of the tile partials
    if (t < n) {
      const int i = t;
      if (i > j) {
        const int Ii = i / 4, ri = i % 4;
        // four interleaved partial sums in a fixed order (short dependent chains)
        const int J0 = (j + 1) / 4;
        const int na = Ii - J0 + 1, total = na + (nb - Ii - 1);
        auto term = [&](int k) {
          return k < na ? partA[4 * tri_pos(Ii, J0 + k, nb) + ri] : partT[4 * tri_pos(Ii + 1 + (k - na), Ii, nb) + ri];
        };
        double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
        int k = 0;
        for (; k + 3 < total; k += 4) {
          s0 += term(k);
          s1 += term(k + 1);
          s2 += term(k + 2);
          s3 += term(k + 3);
        }
        if (k < total) s0 += term(k);
        if (k + 1 < total) s1 += term(k + 1);
        if (k + 2 < total) s2 += term(k + 2);
        pb[i] = beta * ((s0 + s1) + (s2 + s3));
      }
    }
    __syncthreads();
    // (c) updates; K = (beta / 2) p^T v in every warp
    double kk = 0.0;
    for (int i = j + 1 + lane; i < n; i += 32) kk = fma(pb[i], vel(i), kk);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kk += __shfl_xor_sync(0xFFFFFFFFu, kk, o);
    const double K = 0.5 * beta * kk;
    if (actA) {
      double vr[4], wr[4], vc[4], wc[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = 4 * I + r, c = 4 * J + r;
        vr[r] = vel(i);
        wr[r] = i > j ? fma(-K, vr[r], pb[i]) : 0.0;
        vc[r] = vel(c);
        wc[r] = c > j ? fma(-K, vc[r], pb[c]) : 0.0;
      }
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) a[r][c] -= fma(vr[r], wc[c], wr[r] * vc[c]);
      if (J == (j + 1) / 4) publish_col(a, (j + 1) % 4, xn + 4 * I);
    }
    __syncthreads();
  }
  if (isA && I == nb - 1 && J == nb - 1) {
    S.d[n - 2] = a[2][2];
    S.d[n - 1] = a[3][3];
    S.e[n - 2] = a[3][2];
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
      // scale (p_{i-1}, p_i) by 2^-e, e the exponent of the larger one
      const long long bits = __double_as_longlong(fmax(fabs(pm1), fabs(pm2)));
      const int ex = static_cast<int>((bits >> 52) & 0x7FF) - 1023;
      if (ex > -1000) {
        const double sc = __longlong_as_double(static_cast<long long>(1023 - ex) << 52);
        pm1 *= sc;
        pm2 *= sc;
      }
    }
  }
  return cnt;
}

__global__ void __launch_bounds__(32) core_vector_kernel(int n, double* ws, int max_rounds, int32_t* dev_status) {
  __shared__ double d[kMaxN], e[kMaxN], e2[kMaxN], dp[kMaxN], dm[kMaxN], lp[kMaxN], um[kMaxN], z[kMaxN];
  __shared__ __align__(16) double bs[kMaxN];
  extern __shared__ __align__(16) double Vs[];  // n x n reflectors
  __shared__ uint64_t vbar;
  __shared__ int vabort;
  const EigScratch S = scratch(ws, n);
  const int lane = threadIdx.x, idx = blockIdx.x;  // eigenvalue idx in ascending order
  // the reflectors and their betas come in by one bulk copy each, started
  // now so that they land while the eigenvalue is found
  const uint32_t vbytes = static_cast<uint32_t>(n) * n * sizeof(double);
  if (lane == 0) {
    vabort = 0;
    mbar_init(&vbar, 1);
    fence_barrier_init();
    mbar_arrive_expect_tx(&vbar, vbytes + static_cast<uint32_t>(n) * sizeof(double));
    bulk_load(Vs, S.V, vbytes, &vbar);
    bulk_load(bs, S.beta, static_cast<uint32_t>(n) * sizeof(double), &vbar);
  }
  __syncwarp();
  // scale T by a power of two so that |d|, |e| <= 1
  double mx = 0.0;
  for (int i = lane; i < n; i += 32) {
    mx = fmax(mx, fabs(S.d[i]));
    if (i + 1 < n) mx = fmax(mx, fabs(S.e[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  if (mx == 0.0) {  // T = 0: every unit vector is an eigenvector
    for (int i = lane; i < n; i += 32) z[i] = i == idx ? 1.0 : 0.0;
  }
  int ex = 0;
  double lam = 0.0;
  if (mx > 0.0) {
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
    lam = 0.5 * (lo + hi);
    // twisted factorisation of T - lam I: lane 0 runs the top-down LDL^T
    // recurrence, lane 1 the bottom-up UDU^T one at the same time
    const double pivmin = 0x1p-100;
    if (lane == 0) {
      double Dp = d[0] - lam;
      for (int i = 0; i + 1 < n; ++i) {
        if (fabs(Dp) < pivmin) Dp = Dp < 0.0 ? -pivmin : pivmin;
        dp[i] = Dp;
        lp[i] = e[i] / Dp;
        Dp = (d[i + 1] - lam) - lp[i] * e[i];
      }
      dp[n - 1] = Dp;
    } else if (lane == 1) {
      double Dm = d[n - 1] - lam;
      for (int i = n - 1; i > 0; --i) {
        if (fabs(Dm) < pivmin) Dm = Dm < 0.0 ? -pivmin : pivmin;
        dm[i] = Dm;
        um[i - 1] = e[i - 1] / Dm;
        Dm = (d[i - 1] - lam) - um[i - 1] * e[i - 1];
      }
      dm[0] = Dm;
    }
    __syncwarp();
    // twist index r: the smallest |gamma_r| = |D+_r + D-_r - (d_r - lam)|
    // (the lowest r on ties)
    double best = 1e308;
    int r = n;
    for (int i = lane; i < n; i += 32) {
      const double g = fabs(dp[i] + dm[i] - (d[i] - lam));
      if (g < best) {
        best = g;
        r = i;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ob = __shfl_xor_sync(0xFFFFFFFFu, best, o);
      const int orr = __shfl_xor_sync(0xFFFFFFFFu, r, o);
      if (ob < best || (ob == best && orr < r)) {
        best = ob;
        r = orr;
      }
    }
    // z_r = 1; lane 0 walks up, lane 1 walks down (each rescales its own side
    // by 1e-150 if it grows past 1e150; the sides are reconciled after)
    int sc = 0;
    if (lane == 0) {
      for (int i = r - 1; i >= 0; --i) {
        z[i] = -lp[i] * (i + 1 == r ? 1.0 : z[i + 1]);
        if (fabs(z[i]) > 1e150) {
          for (int q = i; q < r; ++q) z[q] *= 1e-150;
          ++sc;
        }
      }
    } else if (lane == 1) {
      for (int i = r; i + 1 < n; ++i) {
        z[i + 1] = -um[i] * (i == r ? 1.0 : z[i]);
        if (fabs(z[i + 1]) > 1e150) {
          for (int q = r + 1; q <= i + 1; ++q) z[q] *= 1e-150;
          ++sc;
        }
      }
    }
    const int s0 = __shfl_sync(0xFFFFFFFFu, sc, 0), s1 = __shfl_sync(0xFFFFFFFFu, sc, 1);
    __syncwarp();
    if (lane == 0) {
      const int smax = s0 > s1 ? s0 : s1;
      double f = 1.0;
      for (int k = 0; k < smax; ++k) f *= 1e-150;
      z[r] = f;
      for (int k = s0; k < smax; ++k)
        for (int q = 0; q < r; ++q) z[q] *= 1e-150;
      for (int k = s1; k < smax; ++k)
        for (int q = r + 1; q < n; ++q) z[q] *= 1e-150;
    }
  }  // mx > 0
  __syncwarp();
  // x = H_0 H_1 ... H_{n-3} z, the reflectors staged in shared memory;
  // lane l holds entries l, l + 32, l + 64, l + 96
  const bool landed = mbar_wait(&vbar, 0, &vabort);  // bounded wait
  if (!__all_sync(0xFFFFFFFFu, landed)) {
    if (lane == 0) {
      report(dev_status, METIS_DEV_TIMEOUT);
      // the copies were issued by this warp: give them a bounded time to land
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(&vbar, 0) && global_timer_ns() - t0 < 100000000ull) {
      }
    }
    __syncwarp();
    return;
  }
  double xv[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) xv[q] = lane + 32 * q < n ? z[lane + 32 * q] : 0.0;
  for (int j = n - 3; j >= 0; --j) {
    const double* vj = Vs + j * n;
    double c = 0.0;
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (lane + 32 * q < n) c = fma(vj[lane + 32 * q], xv[q], c);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
    c *= bs[j];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (lane + 32 * q < n) xv[q] = fma(-c, vj[lane + 32 * q], xv[q]);
  }
  double nrm = 0.0;
#pragma unroll
  for (int q = 0; q < 4; ++q) nrm = fma(xv[q], xv[q], nrm);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) nrm += __shfl_xor_sync(0xFFFFFFFFu, nrm, o);
  const double inv = 1.0 / sqrt(nrm);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (lane + 32 * q < n) S.X[(lane + 32 * q) * n + idx] = xv[q] * inv;
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

__global__ void __launch_bounds__(1024) core_finish_kernel(int n, double* ws, double* eval, float* evec) {
  __shared__ double lam[kMaxN];
  const EigScratch S = scratch(ws, n);
  double* X = S.X;
  for (int i = threadIdx.x; i < n; i += blockDim.x) lam[i] = S.lam[i];
  __syncthreads();
  // is there any cluster at all?  (one warp vote; usually not)
  bool any = false;
  if (threadIdx.x < 32) {
    double top = 0.0;
    for (int i = threadIdx.x; i < n; i += 32) top = fmax(top, fabs(lam[i]));
    for (int o = 16; o > 0; o >>= 1) top = fmax(top, __shfl_xor_sync(0xFFFFFFFFu, top, o));
    const double tol = kClusterTol * top;
    bool gap_small = false;
    for (int i = threadIdx.x; i + 1 < n; i += 32) gap_small |= lam[i + 1] - lam[i] <= tol;
    any = __any_sync(0xFFFFFFFFu, gap_small);
  }
  if (threadIdx.x < 32 && any) {
    double top = 0.0;
    for (int i = 0; i < n; ++i) top = fmax(top, fabs(lam[i]));
    const double tol = kClusterTol * top;
    int c0 = 0, cand = 0;
    while (c0 < n) {
      int c1 = c0 + 1;  // cluster [c0, c1)
      while (c1 < n && lam[c1] - lam[c1 - 1] <= tol) ++c1;
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
#pragma unroll 4
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
    const int r = e / n, rk = e - r * n;
    evec[e] = static_cast<float>(X[r * n + (n - 1 - rk)]);
  }
  for (int i = threadIdx.x; i < n; i += blockDim.x) eval[i] = lam[n - 1 - i];
}

}  // namespace

size_t core_eig_workspace(int n) { return (2 * static_cast<size_t>(n) * n + 4 * n) * sizeof(double); }

void launch_core_eig(double* C, int n, int max_iters, double* eval, float* evec, double* ws, int32_t* dev_status,
                     cudaStream_t s) {
  const int nb = n / 4, nA = nb * (nb + 1) / 2;
  const size_t smem = (3 * static_cast<size_t>(n) + 8 * nA) * sizeof(double);
  if (!ensure_smem(reinterpret_cast<const void*>(core_tridiag_kernel), smem)) return;
  core_tridiag_kernel<<<1, kTriThreads, smem, s>>>(C, n, ws);
  const size_t vsmem = static_cast<size_t>(n) * n * sizeof(double);
  if (!ensure_smem(reinterpret_cast<const void*>(core_vector_kernel), vsmem)) return;
  core_vector_kernel<<<n, 32, vsmem, s>>>(n, ws, max_iters, dev_status);
  core_finish_kernel<<<1, 1024, 0, s>>>(n, ws, eval, evec);
}

}  // namespace metis
