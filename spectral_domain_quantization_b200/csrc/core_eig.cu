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
//      symmetric tridiagonal T (diagonal d, off-diagonal e), keeping the
//      reflectors; A's rows held in registers by thread pairs, two barriers
//      per column.
//   2. core_vector_kernel (one CTA of four warps per eigenvalue): the
//      eigenvalue by multisection on Sturm counts (128 points per round, the
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
// 1. Householder tridiagonalisation
// ---------------------------------------------------------------------------
// Column j: x = A[j+1.., j], alpha = -sign(x0) |x|, v = x - alpha e_1,
// beta = 2 / v^T v, p = beta A' v, K = (beta/2) p^T v, w = p - K v and
// A' -= v w^T + w v^T, which is A' -= q v^T + v p^T with q = p - 2 K v.
// (v, beta) are kept so that the eigenvectors can be taken back through
// H_0 ... H_{n-3} later.
//
// Layout: a thread pair per row.  Thread (i, h) holds the row's columns
// base + 2 r + h (r < NH) in registers, base = j rounded down to even, so
// the two halves shrink together and after every second column the row
// moves one register to the left.  Row warps skip 16-column chunks that lie
// past n and the work of warps whose rows are all finished.  The full
// square is kept (no symmetric packing): the product then needs no
// transposed partial sums.
//
// Two barriers per column:
//   (a) row warps: u = A' x with x0 (not v0) at column j + 1, the sums
//       S1 = sum_{i>j+1} u_i x_i and S2 = sum_{i>j+1} A[i][j+1] x_i, and
//       the values of row j + 1; meanwhile one extra warp sums |x|^2
//       from the per-row squares and finds alpha, beta and v0;
//   (b) all: p_i = beta (u_i + A[i][j+1] (v0 - x0)) and
//       p^T v = p_{j+1} v0 + beta (S1 + (v0 - x0) S2) give K and q; the
//       holders of column j + 1 update it first and write the squares of
//       its entries below the next x0 (the extra warp reduces them);
//   (c) row warps: the rest of the rank-2 update.

template <int NH>
struct TriShared {
  static constexpr int kBuf = 4 * NH + 8;   // row windows reach base + 2 NH - 1 <= n + 2 NH - 4
  static constexpr int kWarps = (4 * NH + 31) / 32;
  // per column parity, by row: .x = x entry of the column, .y = p_i (both 0
  // outside the active rows); the update reads both with one 16-byte load
  double2 xp[2][kBuf];
  double red1a[kWarps], red1b[kWarps];
  double sq[2 * NH];    // by row: x_i^2 of the next column's entries below x0 (0 elsewhere)
  double row1[2];       // row j + 1: u_{j+1} and A[j+1][j+1]
  double refl[2];       // beta, v0 of the current column
};

// Sum of v[0 .. cnt) in a fixed order, two interleaved accumulators.
MDEV double sum_fixed(const double* v, int cnt) {
  double s0 = 0.0, s1 = 0.0;
  int w = 0;
  for (; w + 1 < cnt; w += 2) {
    s0 += v[w];
    s1 += v[w + 1];
  }
  if (w < cnt) s0 += v[w];
  return s0 + s1;
}

MDEV double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// One column step; ODD = j & 1 (registers hold columns base + 2 r + h,
// base = j - ODD).  Warps 0 .. nwr - 1 hold rows; warp nwr the scalars.
template <int NH, int ODD>
MDEV void tri_step(double (&a)[NH], TriShared<NH>& sh, const EigScratch& S, int j, int n, int i, int h,
                   int lane, int warp, int nwr) {
  constexpr int kHoldR = ODD ? 1 : 0;   // register of column j + 1, in thread h = 1 - ODD
  const int hold_h = 1 - ODD;
  const int base = j - ODD;
  double2* cur = sh.xp[j & 1];
  double2* nxt = sh.xp[(j + 1) & 1];
  const bool scalar_warp = warp == nwr;
  if (scalar_warp) {
    // |x|^2 without x0, summed by this warp in a fixed order (the row
    // warps only wrote their rows' squares)
    double sg = 0.0;
    for (int r = lane; r < n; r += 32) sg += sh.sq[r];
    sg = warp_sum(sg);
    const double x0 = cur[j + 1].x;
    double alpha = x0, beta = 0.0, v0 = 0.0;
    if (sg > 0.0) {
      // |x| = s rsqrt(s), s = |x|^2, and beta = 2 / (v0^2 + sg) =
      // 1 / (|x| (|x| + |x0|)): two reciprocal square roots in place of a
      // square root and a division on this warp's chain
      const double s2 = fma(x0, x0, sg);
      const double nrm = s2 * rsqrt(s2);
      alpha = x0 >= 0.0 ? -nrm : nrm;
      v0 = x0 - alpha;                                   // sign(x0) (|x0| + |x|)
      const double r2 = rsqrt(nrm * (nrm + fabs(x0)));
      beta = r2 * r2;
    }
    if (lane == 0) {
      sh.refl[0] = beta;
      sh.refl[1] = v0;
      S.e[j] = alpha;
      S.beta[j] = beta;
    }
  }
  const bool row_ok = !scalar_warp && i < n;
  const bool act = row_ok && i > j;                            // rows of the trailing block
  const bool warp_live = !scalar_warp && 16 * warp + 15 > j;   // some row of the warp is active
  // (a) u_i = sum_c A[i][c] x_c over the row's window
  double u = 0.0;
  if (warp_live) {
    double s[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
    const double2* xw = cur + base + h;
#pragma unroll
    for (int c = 0; c < NH / 8; ++c) {
      if (base + 16 * c < n) {
#pragma unroll
        for (int r = 8 * c; r < 8 * c + 8; ++r) s[r & 7] = fma(a[r], xw[2 * r].x, s[r & 7]);
      }
    }
    u = ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
  }
  u += __shfl_xor_sync(0xFFFFFFFFu, u, 1);
  const double ah = __shfl_sync(0xFFFFFFFFu, a[kHoldR], (lane & ~1) | hold_h);   // A[i][j+1]
  const double xi = act ? cur[i].x : 0.0;
  if (row_ok && i == j && h == ODD) S.d[j] = a[0];
  double s1 = 0.0, s2 = 0.0;
  if (h == 0 && act && i >= j + 2) {
    s1 = u * xi;
    s2 = ah * xi;
  }
  if (h == 0 && row_ok && i == j + 1) {
    sh.row1[0] = u;
    sh.row1[1] = ah;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, o);
    s2 += __shfl_xor_sync(0xFFFFFFFFu, s2, o);
  }
  if (lane == 0 && !scalar_warp) {
    sh.red1a[warp] = s1;
    sh.red1b[warp] = s2;
  }
  __syncthreads();
  // (b) p, K, q; column j + 1 and the next |x|^2
  const double beta = sh.refl[0], v0 = sh.refl[1];
  const double dv = v0 - cur[j + 1].x;
  const double S1 = sum_fixed(sh.red1a, nwr), S2 = sum_fixed(sh.red1b, nwr);
  const double pj1 = beta * fma(sh.row1[1], dv, sh.row1[0]);
  const double K = 0.5 * beta * fma(pj1, v0, beta * fma(dv, S2, S1));
  const double pi = act ? beta * fma(ah, dv, u) : 0.0;
  const double vi = !act ? 0.0 : (i == j + 1 ? v0 : xi);
  const double qi = fma(-2.0 * K, vi, pi);
  if (h == 0 && row_ok) {
    cur[i].y = pi;
    S.V[j * n + i] = beta == 0.0 ? 0.0 : vi;
    if (i <= j + 1) nxt[i].x = 0.0;
  }
  if (h == hold_h && row_ok) {
    a[kHoldR] = fma(-qi, v0, fma(-vi, pj1, a[kHoldR]));
    if (i >= j + 2) nxt[i].x = a[kHoldR];
    sh.sq[i] = i >= j + 3 ? a[kHoldR] * a[kHoldR] : 0.0;
  }
  __syncthreads();
  // (c) the rest of the update: a_ic -= q_i v_c + v_i p_c (v_c = x_c past
  // column j + 1, whose register was updated above)
  if (warp_live) {
    const double2* xw = cur + base + h;
#pragma unroll
    for (int c = 0; c < NH / 8; ++c) {
      if (base + 16 * c < n) {
#pragma unroll
        for (int r = 8 * c; r < 8 * c + 8; ++r) {
          if (h == hold_h && r == kHoldR) continue;
          const double2 xpc = xw[2 * r];
          a[r] = fma(-qi, xpc.x, fma(-vi, xpc.y, a[r]));
        }
      }
    }
  }
}

// One CTA of round32(2 n) + 32 threads, n <= 2 NH.
template <int NH>
__global__ void __launch_bounds__(4 * NH + 32, 1) core_tridiag_kernel(const double* C, int n, double* ws) {
  __shared__ TriShared<NH> sh;
  const EigScratch S = scratch(ws, n);
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int nwr = (blockDim.x >> 5) - 1;
  const int i = t >> 1, h = t & 1;
  const bool row_ok = warp < nwr && i < n;
  double a[NH];
#pragma unroll
  for (int r = 0; r < NH; ++r) {
    const int c = 2 * r + h;
    a[r] = (row_ok && c < n) ? C[i * n + c] : 0.0;
  }
  for (int e = t; e < 2 * TriShared<NH>::kBuf; e += blockDim.x) (&sh.xp[0][0])[e] = make_double2(0.0, 0.0);
  __syncthreads();
  {
    // column 0: x_i = A[i][0] (i >= 1) and |x|^2 without x0
    if (h == 0 && row_ok && i >= 1) sh.xp[0][i].x = a[0];
    if (h == 0 && row_ok) sh.sq[i] = i >= 2 ? a[0] * a[0] : 0.0;
    __syncthreads();
  }
  int j = 0;
  bool even_next = true;   // registers hold base = j
  while (j + 2 < n) {
    tri_step<NH, 0>(a, sh, S, j, n, i, h, lane, warp, nwr);
    ++j;
    even_next = false;
    if (j + 2 >= n) break;
    tri_step<NH, 1>(a, sh, S, j, n, i, h, lane, warp, nwr);
    if (warp < nwr && 16 * warp + 15 > j) {
      // move the row one register left (chunks past n hold zeros already)
#pragma unroll
      for (int c = 0; c < NH / 8; ++c) {
        if (j - 1 + 16 * c < n) {
#pragma unroll
          for (int r = 8 * c; r < 8 * c + 8; ++r) a[r] = r + 1 < NH ? a[r + 1] : 0.0;
        }
      }
    }
    ++j;
    even_next = true;
  }
  if (!row_ok) return;
  if (n == 1) {
    S.d[0] = a[0];
    return;
  }
  // the last 2 x 2 block, columns n - 2 and n - 1
  if (even_next) {   // base = n - 2: column n - 2 in (h 0, r 0), n - 1 in (h 1, r 0)
    if (i == n - 2 && h == 0) S.d[n - 2] = a[0];
    if (i == n - 1 && h == 0) S.e[n - 2] = a[0];
    if (i == n - 1 && h == 1) S.d[n - 1] = a[0];
  } else {           // base = n - 3: column n - 2 in (h 1, r 0), n - 1 in (h 0, r 1)
    if (i == n - 2 && h == 1) S.d[n - 2] = a[0];
    if (i == n - 1 && h == 1) S.e[n - 2] = a[0];
    if (i == n - 1 && h == 0) S.d[n - 1] = a[1];
  }
}

template <int NH>
void launch_tridiag(const double* C, int n, double* ws, cudaStream_t s) {
  const int threads = (2 * n + 31) / 32 * 32 + 32;
  core_tridiag_kernel<NH><<<1, threads, 0, s>>>(C, n, ws);
}

// ---------------------------------------------------------------------------
// 2. one eigenpair per CTA (one warp)
// ---------------------------------------------------------------------------

// Sign of p as -1 / +1, or `prev` for a zero (bit tests: the fp64 compare
// unit is far slower than the integer pipe).
MDEV int sign_or(double p, int prev) {
  const long long b = __double_as_longlong(p);
  return (b << 1) == 0 ? prev : (b < 0 ? -1 : 1);
}

// Biased exponent field of |p|.
MDEV int exp_field(double p) { return static_cast<int>((__double_as_longlong(p) >> 52) & 0x7FF); }

// Number of eigenvalues of T below x (scaled T: |d|, |e| <= 1): sign changes
// of the leading principal minors p_{-1} = 1, p_0, ..., p_{n-1}, with
// p_i = (d_i - x) p_{i-1} - e_{i-1}^2 p_{i-2}; a zero minor takes the sign of
// the one before it.  The pair (p_{i-1}, p_i) is rescaled by a power of two
// every fourth step (|p| grows at most 5x per step), so nothing overflows.
MDEV int sturm_count(const double* d, const double* e2, int n, double x) {
  double pm2 = 1.0, pm1 = d[0] - x;
  int sg = sign_or(pm1, 1);
  int cnt = sg != 1;
  // four steps per pass, their loads issued together ahead of the recurrence
  // (only the fma on p_{i-1} is on the dependent chain)
  int i = 1;
  for (; i + 3 < n; i += 4) {
    double dd[4], ff[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      dd[u] = d[i + u] - x;
      ff[u] = e2[i + u - 1];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const double p = fma(dd[u], pm1, -ff[u] * pm2);
      const int sv = sign_or(p, sg);
      cnt += sv != sg;
      sg = sv;
      pm2 = pm1;
      pm1 = p;
    }
    // scale (p_{i-1}, p_i) by 2^-e, e the exponent of the larger one (a
    // power of two: the signs, and so the count, are unchanged)
    const int ef = max(exp_field(pm1), exp_field(pm2));
    const int ex = ef - 1023;
    if (ex > -1000) {
      const double sc = __longlong_as_double(static_cast<long long>(1023 - ex) << 52);
      pm1 *= sc;
      pm2 *= sc;
    }
  }
  for (; i < n; ++i) {
    const double p = fma(d[i] - x, pm1, -e2[i - 1] * pm2);
    const int sv = sign_or(p, sg);
    cnt += sv != sg;
    sg = sv;
    pm2 = pm1;
    pm1 = p;
  }
  return cnt;
}

constexpr int kVecWarps = 4;   // warps per eigenvalue CTA

__global__ void __launch_bounds__(32 * kVecWarps) core_vector_kernel(int n, double* ws, int max_rounds,
                                                                     int32_t* dev_status) {
  __shared__ double d[kMaxN], e[kMaxN], e2[kMaxN], dp[kMaxN], dm[kMaxN], lp[kMaxN], um[kMaxN], z[kMaxN];
  __shared__ __align__(16) double bs[kMaxN];
  extern __shared__ __align__(16) double Vs[];  // n x n reflectors
  __shared__ uint64_t vbar;
  __shared__ int vabort;
  __shared__ double interval[2];                // the Gershgorin interval, by warp 0
  __shared__ int scaled;                        // T != 0 (the multisection runs)
  __shared__ unsigned masks[2][kVecWarps];      // per round parity: each warp's ballot
  __shared__ double part[2][kVecWarps];         // per step parity: each warp's partial dot product
  const EigScratch S = scratch(ws, n);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int idx = blockIdx.x;  // eigenvalue idx in ascending order
  // the reflectors and their betas come in by one bulk copy each, started
  // now so that they land while the eigenvalue is found
  const uint32_t vbytes = static_cast<uint32_t>(n) * n * sizeof(double);
  if (tid == 0) {
    vabort = 0;
    mbar_init(&vbar, 1);
    fence_barrier_init();
    mbar_arrive_expect_tx(&vbar, vbytes + static_cast<uint32_t>(n) * sizeof(double));
    bulk_load(Vs, S.V, vbytes, &vbar);
    bulk_load(bs, S.beta, static_cast<uint32_t>(n) * sizeof(double), &vbar);
  }
  int ex = 0;
  if (warp == 0) {
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
    } else {
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
      if (lane == 0) {
        interval[0] = lo - 1e-12;
        interval[1] = hi + 1e-12;
      }
    }
    if (lane == 0) scaled = mx > 0.0;
  }
  __syncthreads();
  double lam = 0.0;   // found by warp 0 (thread 0 writes it with warp 0's exponent ex)
  if (scaled) {
    // multisection over all warps: point t = 32 w + l (0 .. 127) sits at
    // lo + (hi - lo) (t + 1) / 129, rising with t; the smallest point with
    // count > idx bounds the eigenvalue.  Every thread updates (lo, hi) from
    // the four ballots by the same float operations, so they stay equal.
    constexpr int kPoints = 32 * kVecWarps;
    double lo = interval[0], hi = interval[1];
    bool done = false;
    for (int round = 0; round < max_rounds; ++round) {
      if (hi - lo <= 0x1p-50 * fmax(fabs(lo), fabs(hi)) + 0x1p-60) {
        done = true;
        break;
      }
      const double w = hi - lo;
      const double x = lo + w * (static_cast<double>(tid + 1) / (kPoints + 1));
      const int c = sturm_count(d, e2, n, x);
      const unsigned mask = __ballot_sync(0xFFFFFFFFu, c > idx);
      if (lane == 0) masks[round & 1][warp] = mask;
      __syncthreads();
      int f = kPoints;  // the first point with count > idx
#pragma unroll
      for (int q = kVecWarps - 1; q >= 0; --q) {
        const unsigned mq = masks[round & 1][q];
        if (mq) f = 32 * q + __ffs(mq) - 1;
      }
      const double nlo = f > 0 ? lo + w * (static_cast<double>(f) / (kPoints + 1)) : lo;
      if (f < kPoints) hi = lo + w * (static_cast<double>(f + 1) / (kPoints + 1));
      lo = nlo;
    }
    if (!done && tid == 0) report(dev_status, METIS_DEV_NUMERIC);
    if (warp == 0) {
      lam = 0.5 * (lo + hi);
      // twisted factorisation of T - lam I: lane 0 runs the top-down LDL^T
      // recurrence, lane 1 the bottom-up UDU^T one, in lockstep (one
      // instruction stream, per-lane indices)
      const double pivmin = 0x1p-100;
      if (lane < 2) {
        // the chain per step is one reciprocal and one fma: the pivot guard
        // reads the exponent bits (|D| < 2^-100), the multiplier l = e / D
        // and D' = (d - lam) - e^2 / D come from 1 / D, and the loads and
        // stores (restrict: the arrays do not overlap) leave the chain
        const bool up = lane == 1;
        double* __restrict__ Dst = up ? dm : dp;
        double* __restrict__ Lst = up ? um : lp;
        const double* __restrict__ dd = d;
        const double* __restrict__ ev = e;
        const double* __restrict__ ev2 = e2;
        double D = (up ? dd[n - 1] : dd[0]) - lam;
        for (int st = 0; st + 1 < n; ++st) {
          const int ie = up ? n - 2 - st : st;      // e index of this step
          const int inext = up ? n - 2 - st : st + 1;
          const double ee = ev[ie], ee2 = ev2[ie], dn = dd[inext] - lam;
          if (exp_field(D) < 1023 - 100) D = __double_as_longlong(D) < 0 ? -pivmin : pivmin;
          Dst[up ? n - 1 - st : st] = D;
          const double rD = 1.0 / D;
          Lst[ie] = ee * rD;
          D = fma(-ee2, rD, dn);
        }
        Dst[up ? 0 : n - 1] = D;
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
      if (r >= n) r = 0;  // no finite gamma (a non-finite input): any in-range twist
      // z_r = 1; lane 0 walks up, lane 1 walks down, in lockstep (each
      // rescales its own side by 1e-150 once |z| reaches 2^499 (about
      // 1.6e150; read from the exponent bits); the sides are reconciled
      // after).  restrict: the multipliers and z do not overlap, so the
      // multiplier loads leave the chain.
      int sc = 0;
      if (lane < 2) {
        const bool up = lane == 0;
        const double* __restrict__ mul = up ? lp : um;
        double* __restrict__ zz = z;
        const int steps = up ? r : n - 1 - r;
        const int smax = r > n - 1 - r ? r : n - 1 - r;
        double zc = 1.0;
        for (int st = 0; st < smax; ++st) {
          if (st < steps) {
            const int i = up ? r - 1 - st : r + st;      // multiplier index
            const int dst = up ? r - 1 - st : r + 1 + st;
            zc = -mul[i] * zc;
            zz[dst] = zc;
            if (exp_field(zc) > 1023 + 498) {
              const int q0 = up ? dst : r + 1, q1 = up ? r - 1 : dst;
              for (int q = q0; q <= q1; ++q) zz[q] *= 1e-150;   // through zz: the one name for z here
              zc *= 1e-150;
              ++sc;
            }
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
    }
  }
  __syncthreads();
  // x = H_0 H_1 ... H_{n-3} z, the reflectors staged in shared memory;
  // thread t holds entry t (n <= 128); each reflector's dot product is a
  // warp reduction, then the four warp sums in warp order
  const bool landed = mbar_wait(&vbar, 0, &vabort);  // bounded wait
  if (!__syncthreads_and(landed)) {
    if (tid == 0) {
      report(dev_status, METIS_DEV_TIMEOUT);
      // the copies were issued by this CTA: give them a bounded time to land
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(&vbar, 0) && global_timer_ns() - t0 < 100000000ull) {
      }
    }
    __syncthreads();
    return;
  }
  const bool mine = tid < n;
  double xv = mine ? z[tid] : 0.0;
  int par = 0;
  for (int j = n - 3; j >= 0; --j, par ^= 1) {
    const double vt = mine ? Vs[j * n + tid] : 0.0;
    double c = vt * xv;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
    if (lane == 0) part[par][warp] = c;
    __syncthreads();
    c = ((part[par][0] + part[par][1]) + (part[par][2] + part[par][3])) * bs[j];
    xv = fma(-c, vt, xv);
  }
  double nrm = xv * xv;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) nrm += __shfl_xor_sync(0xFFFFFFFFu, nrm, o);
  if (lane == 0) part[par][warp] = nrm;
  __syncthreads();
  nrm = (part[par][0] + part[par][1]) + (part[par][2] + part[par][3]);
  const double inv = 1.0 / sqrt(nrm);
  if (mine) S.X[tid * n + idx] = xv * inv;
  if (tid == 0) S.lam[idx] = ldexp(lam, ex);
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
  if (n <= 32) launch_tridiag<16>(C, n, ws, s);
  else if (n <= 48) launch_tridiag<24>(C, n, ws, s);
  else if (n <= 80) launch_tridiag<40>(C, n, ws, s);
  else launch_tridiag<56>(C, n, ws, s);
  const size_t vsmem = static_cast<size_t>(n) * n * sizeof(double);
  if (!ensure_smem(reinterpret_cast<const void*>(core_vector_kernel), vsmem)) return;
  core_vector_kernel<<<n, 32 * kVecWarps, vsmem, s>>>(n, ws, max_iters, dev_status);
  core_finish_kernel<<<1, 1024, 0, s>>>(n, ws, eval, evec);
}

}  // namespace metis
