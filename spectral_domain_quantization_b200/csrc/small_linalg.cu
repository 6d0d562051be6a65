// Small dense linear algebra of the randomized split (l = k + p <= 112):
// Gram matrices, Cholesky with rank drop and forward substitution (CholeskyQR),
// row-block products, factor assembly and the sign convention.  The core's
// eigen-decomposition lives in core_eig.cu.
//
// Source: SII release on Metis, section 2.4 item 1 (spectral decomposition in
// a low-dimensional space after randomized reduction); older Metis abstract
// item (i) (random embedding separates dominant from long-tail parts).
//
// Numerics: Gram matrices are accumulated in float64 from float32 rows;
// the Cholesky factor runs in float64 in one CTA; tall row blocks are
// multiplied (or solved against the factor) in float32.
//   * CholeskyQR: G = Y^T Y = L L^T, Q = Y L^-T.  A pivot that falls below
//     1e-12 of its original diagonal (a numerically dependent sketch column,
//     e.g. for an exactly low-rank input) is dropped: that column of Q
//     becomes zero instead of amplified rounding noise.
#include "common.cuh"
#include "abi_common.h"
#include "small_linalg.h"

namespace metis {

namespace {

constexpr double kDropTol = 1e-12;

// Gram partial of a row block held in shared memory (rows x cols values of
// type T with row stride ld, cols a multiple of 4): the upper 4 x 4 tiles
// (bi <= bj), tile p written as 16 contiguous doubles out[16 p + 4 x + y] =
// sum_r Y[r][4 bi + x] Y[r][4 bj + y], p counting the pairs bi-major.  Each
// thread accumulates one tile (16 independent float64 chains).
template <typename T>
MDEV void gram_block(const T* ys, int rows, int cols, int ld, double* out) {
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
#pragma unroll 4
    for (int r = 0; r < rows; ++r) {
      const T* row = ys + r * ld;
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
    double* o = out + 16 * pidx;
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int y = 0; y < 4; ++y) o[4 * x + y] = acc[x][y];
  }
}

constexpr int kGramRows = 32;

// Float64 Gram partial of each 32-row block of Y (rows x lp float32, row
// stride lp): the block staged in shared memory as float64 (each value
// converted once), then 4 x 4 register tiles over the rows in order.  One
// thread per 4 x 4 tile pair (blockDim covers (lp/4)(lp/4+1)/2 pairs).
__global__ void __launch_bounds__(1024) gram_kernel(const float* __restrict__ Y, int64_t rows, int lp,
                                                    double* __restrict__ gpart) {
  extern __shared__ double ys[];  // kGramRows x (lp + 1)
  const int ld = lp + 1;
  const int q4 = lp / 4;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kGramRows;
  const int nr = static_cast<int>(imin64(kGramRows, rows - r0));
  for (int e = threadIdx.x; e < kGramRows * q4; e += blockDim.x) {
    const int r = e / q4, c4 = e - r * q4;
    const float4 x = r < nr ? reinterpret_cast<const float4*>(Y)[(r0 + r) * q4 + c4] : make_float4(0.f, 0.f, 0.f, 0.f);
    double* d = ys + r * ld + 4 * c4;
    d[0] = x.x;
    d[1] = x.y;
    d[2] = x.z;
    d[3] = x.w;
  }
  __syncthreads();
  gram_block(ys, nr, lp, ld, gpart + static_cast<int64_t>(blockIdx.x) * lp * lp);
}

// Sum of the block partials (packed upper tiles, block stride lp^2): a CTA
// takes 32 consecutive packed entries (coalesced 256-byte runs of each
// partial); its 8 warps take every 8th block, the 8 sums are added in warp
// order (deterministic), and each entry goes to G[i][j] and G[j][i].
constexpr int kReduceGroups = 8;
__global__ void __launch_bounds__(256) gram_reduce_kernel(const double* __restrict__ gpart, int nblocks, int lp,
                                                          double* __restrict__ G) {
  __shared__ double part[kReduceGroups][32];
  const int lane = threadIdx.x & 31, grp = threadIdx.x >> 5;
  const int nb = lp / 4;
  const int npk = 8 * nb * (nb + 1);   // packed entries: 16 per tile pair
  const int e = blockIdx.x * 32 + lane;
  const int64_t stride = static_cast<int64_t>(lp) * lp;
  double s = 0.0;
  if (e < npk) {
#pragma unroll 8
    for (int b = grp; b < nblocks; b += kReduceGroups) s += gpart[static_cast<int64_t>(b) * stride + e];
  }
  part[grp][lane] = s;
  __syncthreads();
  if (grp == 0 && e < npk) {
    double t = 0.0;
#pragma unroll
    for (int g = 0; g < kReduceGroups; ++g) t += part[g][lane];
    int pidx = e >> 4, bi = 0;
    while (pidx >= nb - bi) {
      pidx -= nb - bi;
      ++bi;
    }
    const int bj = bi + pidx, x = (e >> 2) & 3, y = e & 3;
    const int i = 4 * bi + x, j = 4 * bj + y;
    G[i * lp + j] = t;
    G[j * lp + i] = t;
  }
}

// column 1 ...) of an n x n matrix, packed as (row << 8) | column.
MDEV int tri_element(int e, int n) {
  const int ntri = n * (n + 1) / 2;
  const int er = ntri - 1 - e;  // index counted from the last element
  // w = length of the column holding er counted from the right: the smallest
  // w with w (w + 1) / 2 > er
  int w = static_cast<int>((sqrtf(8.f * er + 1.f) - 1.f) * 0.5f) + 1;
  while (w * (w + 1) / 2 <= er) ++w;
  while (w > 1 && (w - 1) * w / 2 > er) --w;
  const int c = n - w;
  const int i = n - 1 - (er - (w - 1) * w / 2);
  return (i << 8) | c;
}

constexpr int kSmallThreads = 512;
constexpr int kTile = 4;  // register tile edge and panel width of the Cholesky
// Panel buffer layout: tile row I (rows 4I .. 4I+3, 4 columns: 16 doubles)
// starts at double 18 I.  The 16-byte skew puts the same word of consecutive
// tile rows in different bank groups: the warps' 16-byte reads of their own
// tile rows then run at the minimum 4 wavefronts instead of up to 32.
constexpr int kPanStride = 18;

// Factor the diagonal tile (K, K), held in registers by its owner (lower
// triangle valid), in place: column c takes the pivot d = v[c][c], dropped
// (1/sqrt = 0, the column of L zero) when it falls below kDropTol of its
// original diagonal; otherwise L[a][c] = v[a][c] / sqrt(d) and the columns
// right of it take the rank-1 update.  Writes L's diagonal block, 1/sqrt(d)
// and sqrt(d).
MDEV void factor_diag(double (&v)[kTile][kTile], int K, double* L, double* invd, double* sqd, const double* diag0,
                      int ld) {
  const int o = kTile * K;
#pragma unroll
  for (int c = 0; c < kTile; ++c) {
    const double d = v[c][c];
    const bool drop = !(diag0[o + c] > 0.0) || !(d > kDropTol * diag0[o + c]);
    const double ri = drop ? 0.0 : rsqrt(d);
    invd[o + c] = ri;
    sqd[o + c] = d * ri;
    double l[kTile];
#pragma unroll
    for (int a = 0; a < kTile; ++a) l[a] = a > c ? v[a][c] * ri : 0.0;
#pragma unroll
    for (int a = c + 1; a < kTile; ++a)
#pragma unroll
      for (int b = c + 1; b <= a; ++b) v[a][b] = fma(-l[a], l[b], v[a][b]);
#pragma unroll
    for (int a = 0; a < kTile; ++a) L[(o + a) * ld + o + c] = a == c ? d * ri : l[a];
  }
}

// Rows 4I .. 4I+3 of panel K (the owner's updated tile (I, K), I > K):
// forward substitution with the panel's diagonal block of L,
// L[r][c] = (v[r][c] - sum_{c' < c} L[r][c'] L[c][c']) / sqrt(pivot c), into
// the panel buffer P (lp x 4) and L.
MDEV void solve_rows(const double (&v)[kTile][kTile], int I, int K, double* P, double* L, const double* invd, int ld) {
  const int o = kTile * K;
  double dl[kTile][kTile], ri[kTile];
#pragma unroll
  for (int c = 0; c < kTile; ++c) {
    ri[c] = invd[o + c];
#pragma unroll
    for (int cp = 0; cp < c; ++cp) dl[c][cp] = L[(o + c) * ld + o + cp];
  }
#pragma unroll
  for (int a = 0; a < kTile; ++a) {
    double lr[kTile];
#pragma unroll
    for (int c = 0; c < kTile; ++c) {
      double x = v[a][c];
#pragma unroll
      for (int cp = 0; cp < c; ++cp) x = fma(-lr[cp], dl[c][cp], x);
      lr[c] = x * ri[c];
    }
    const int row = kTile * I + a;
#pragma unroll
    for (int c = 0; c < kTile; ++c) {
      P[I * kPanStride + a * kTile + c] = lr[c];
      L[row * ld + o + c] = lr[c];
    }
  }
}

// Rank-4 update of the register tile (I, J) with panel P: v -= L(I, K) L(J, K)^T.
MDEV void panel_update(double (&v)[kTile][kTile], const double* P, int I, int J) {
  double li[kTile][kTile], lj[kTile][kTile];
  const double2* pi = reinterpret_cast<const double2*>(P + I * kPanStride);
  const double2* pj = reinterpret_cast<const double2*>(P + J * kPanStride);
#pragma unroll
  for (int a = 0; a < kTile; ++a)
#pragma unroll
    for (int c = 0; c < kTile; c += 2) {
      const double2 x = pi[a * 2 + c / 2], y = pj[a * 2 + c / 2];
      li[a][c] = x.x;
      li[a][c + 1] = x.y;
      lj[a][c] = y.x;
      lj[a][c + 1] = y.y;
    }
#pragma unroll
  for (int a = 0; a < kTile; ++a)
#pragma unroll
    for (int b = 0; b < kTile; ++b) {
      double s = v[a][b];
#pragma unroll
      for (int c = 0; c < kTile; ++c) s = fma(-li[a][c], lj[b][c], s);
      v[a][b] = s;
    }
}

// G = L L^T (with drops), written column by column for solve_kernel.
//  Cholesky, right-looking by panels of 4 columns with look-ahead: thread
//  32 + T owns the 4 x 4 tile (I, J), I >= J, of the lower triangle in
//  registers; panel K's columns of L sit in shared memory.  Per panel K + 1,
//  two barriers:
//    (A) every tile right of panel K takes its rank-4 update; the owner of
//        the diagonal tile (K+1, K+1) then factors it at once;
//    (B) the owners of the tiles below it solve their rows of panel K + 1.
//  The float64 factor is then written as float32 column by column, the
//  diagonal as the reciprocal pivots: Lt[i][i] = 1 / L[i][i] (0 for a
//  dropped pivot), Lt[i][m] = L[m][i] for m > i, 0 above.  (An explicit
//  inverse by 16 x 16 blocks took a third of this kernel's time, more than
//  the forward substitution that replaces it costs in solve_kernel.)
__global__ void __launch_bounds__(kSmallThreads, 1) cholesky_kernel(const double* G, int lp, float* Lt) {
  extern __shared__ double sm[];
  const int ld = lp + 1;
  double* pan = sm;               // 2 panel buffers of (lp / 4) x kPanStride
  const int pan_size = (lp / kTile) * kPanStride;
  double* invd = pan + 2 * pan_size;  // lp: 1/sqrt(pivot) (0 when dropped)
  double* sqd = invd + lp;        // lp: sqrt(pivot) (0 when dropped)
  double* diag0 = sqd + lp;       // lp: the original diagonal (drop rule)
  double* L = diag0 + lp;         // lp x ld: final L
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int nb = lp / kTile;
  const int ntiles = nb * (nb + 1) / 2;
  int I = 0, J = 0;
  double v[kTile][kTile];
  const bool owner = t >= 32 && t - 32 < ntiles;
  if (owner) {
    const int ij = tri_element(t - 32, nb);
    I = ij >> 8;
    J = ij & 255;
#pragma unroll
    for (int a = 0; a < kTile; ++a)
#pragma unroll
      for (int b = 0; b < kTile; ++b) v[a][b] = G[(kTile * I + a) * lp + kTile * J + b];
    if (I == J) {
#pragma unroll
      for (int a = 0; a < kTile; ++a) diag0[kTile * I + a] = v[a][a];
    }
  }
  __syncthreads();
  if (owner && I == 0 && J == 0) factor_diag(v, 0, L, invd, sqd, diag0, ld);
  __syncthreads();
  if (owner && J == 0 && I > 0) solve_rows(v, I, 0, pan, L, invd, ld);
  __syncthreads();
  for (int K = 0; K + 1 < nb; ++K) {
    const double* P = pan + (K & 1) * pan_size;
    double* Pn = pan + ((K + 1) & 1) * pan_size;
    if (owner && J > K) {
      panel_update(v, P, I, J);
      if (I == K + 1 && J == K + 1) factor_diag(v, K + 1, L, invd, sqd, diag0, ld);
    }
    __syncthreads();
    if (owner && J == K + 1 && I > K + 1) solve_rows(v, I, K + 1, Pn, L, invd, ld);
    __syncthreads();
  }
  for (int i = warp; i < lp; i += kSmallThreads / 32)
    for (int m = lane; m < lp; m += 32)
      Lt[i * lp + m] = m > i ? static_cast<float>(L[m * ld + i]) : (m == i ? static_cast<float>(invd[i]) : 0.f);
}

constexpr int kApplyRows = 32;

// out = in (rows x kin) * M (kin x kout).  32 rows per CTA, 256 threads, each
// thread a 4-row x 4-column register tile (4 consecutive columns).  Optional fp32 out,
// transposed bf16 hi/lo copy, Gram partial of the output block, and per
// column the block's largest |out| with its first row (the sign convention).
MDEV void apply_store(const ApplyArgs& a, int64_t blk, int64_t r0, int nr, const float* Out);

MDEV void apply_block(const ApplyArgs& a, int64_t blk) {
  extern __shared__ float smf[];
  float* Ms = smf;                                   // kin x kout
  float* In = Ms + a.kin * a.kout;                   // kApplyRows x (kin + 1)
  float* Out = In + kApplyRows * (a.kin + 1);        // kApplyRows x (kout + 1)
  const int64_t r0 = blk * kApplyRows;
  const int nr = static_cast<int>(imin64(kApplyRows, a.rows - r0));
  {
    const float4* M4 = reinterpret_cast<const float4*>(a.M);
    float4* Ms4 = reinterpret_cast<float4*>(Ms);
    const int n4 = a.kin * a.kout / 4;
#pragma unroll 8
    for (int e = threadIdx.x; e < n4; e += blockDim.x) Ms4[e] = M4[e];
    const int q4 = a.kin / 4;
#pragma unroll 4
    for (int e = threadIdx.x; e < kApplyRows * q4; e += blockDim.x) {
      const int r = e / q4, c4 = e - r * q4;
      const float4 x = r < nr ? *reinterpret_cast<const float4*>(a.in + (r0 + r) * a.in_ld + 4 * c4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
      float* d = In + r * (a.kin + 1) + 4 * c4;
      d[0] = x.x;
      d[1] = x.y;
      d[2] = x.z;
      d[3] = x.w;
    }
  }
  __syncthreads();
  // thread t < 8 kout / 4: rows 4 rg .. 4 rg + 3 (broadcast reads of In) and
  // columns 4 cg .. 4 cg + 3 (one 16-byte read of M per step), rg = t / (kout
  // / 4), cg = t % (kout / 4): every lane of the first warps works (kout <= 112)
  const int ncg = a.kout / 4;
  const int t = threadIdx.x;
  const bool has = t < 8 * ncg;
  const int rg = has ? t / ncg : 0, cg = has ? t - rg * ncg : 0;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[i][u] = 0.f;
  const float* in0 = In + (4 * rg) * (a.kin + 1);
  if (has) {
#pragma unroll 2
    for (int j = 0; j < a.kin; ++j) {
      float x[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) x[i] = in0[i * (a.kin + 1) + j];
      const float4 m = *reinterpret_cast<const float4*>(Ms + j * a.kout + 4 * cg);
      const float mv[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i][u] = fmaf(x[i], mv[u], acc[i][u]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int u = 0; u < 4; ++u) Out[(4 * rg + i) * (a.kout + 1) + 4 * cg + u] = acc[i][u];
  }
  __syncthreads();
  apply_store(a, blk, r0, nr, Out);
}

// The stores of one 32-row block from its result rows in shared memory
// (Out, row stride kout + 1): fp32 rows, the bf16 hi / lo transpose, the
// Gram partial and the per-column block maxima, each where requested.
MDEV void apply_store(const ApplyArgs& a, int64_t blk, int64_t r0, int nr, const float* Out) {
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
  if (a.gpart) gram_block<float>(Out, nr, a.kout, a.kout + 1, a.gpart + blk * a.kout * a.kout);
  if (a.bmax && threadIdx.x < a.kout) {
    // rows in order, strictly larger wins (the lowest row on ties); a NaN
    // never wins, so a column of NaNs keeps -1 and the block's first row
    const int j = threadIdx.x;
    float best = -1.f;
    int64_t bi = r0;
    for (int r = 0; r < nr; ++r) {
      const float v = fabsf(Out[r * (a.kout + 1) + j]);
      if (v > best) {
        best = v;
        bi = r0 + r;
      }
    }
    a.bmax[blk * a.kout + j] = best;
    a.bidx[blk * a.kout + j] = bi;
  }
}

__global__ void __launch_bounds__(256) apply_kernel(ApplyArgs a) { apply_block(a, blockIdx.x); }

// out = in L^-T for the lower-triangular Cholesky factor L (KIN x KIN), by
// forward substitution row by row: L q^T = y^T, q_i = (y_i - sum_{m<i}
// L[i][m] q_m) / L[i][i].  M holds L column by column with the reciprocal
// pivots on the diagonal: M[i][i] = 1 / L[i][i] (0 for a dropped pivot, so
// that column of the result is 0), M[i][m] = L[m][i] below it.  A thread
// takes one row of the 32-row block, its KIN running values in registers
// (right-looking: once q_i is known, every later value takes its term).
template <int KIN>
__global__ void __launch_bounds__(256) solve_kernel(ApplyArgs a) {
  extern __shared__ float smf[];
  float* Ms = smf;                                   // KIN x KIN
  float* In = Ms + KIN * KIN;                        // kApplyRows x (KIN + 1)
  float* Out = In + kApplyRows * (KIN + 1);          // kApplyRows x (KIN + 1)
  const int64_t blk = blockIdx.x;
  const int64_t r0 = blk * kApplyRows;
  const int nr = static_cast<int>(imin64(kApplyRows, a.rows - r0));
  {
    const float4* M4 = reinterpret_cast<const float4*>(a.M);
    float4* Ms4 = reinterpret_cast<float4*>(Ms);
#pragma unroll 4
    for (int e = threadIdx.x; e < KIN * KIN / 4; e += blockDim.x) Ms4[e] = M4[e];
    constexpr int q4 = KIN / 4;
    for (int e = threadIdx.x; e < kApplyRows * q4; e += blockDim.x) {
      const int r = e / q4, c4 = e - r * q4;
      const float4 x = r < nr ? *reinterpret_cast<const float4*>(a.in + (r0 + r) * a.in_ld + 4 * c4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
      float* d = In + r * (KIN + 1) + 4 * c4;
      d[0] = x.x;
      d[1] = x.y;
      d[2] = x.z;
      d[3] = x.w;
    }
  }
  __syncthreads();
  if (threadIdx.x < kApplyRows) {
    const int r = threadIdx.x;
    float acc[KIN];
#pragma unroll
    for (int c = 0; c < KIN; ++c) acc[c] = In[r * (KIN + 1) + c];
#pragma unroll
    for (int i = 0; i < KIN; ++i) {
      const float* col = Ms + i * KIN;
      const float q = acc[i] * col[i];
      acc[i] = q;
#pragma unroll
      for (int m4 = (i + 1) / 4; m4 < KIN / 4; ++m4) {
        const float4 l = reinterpret_cast<const float4*>(col)[m4];
        if (4 * m4 + 0 > i) acc[4 * m4 + 0] = fmaf(-l.x, q, acc[4 * m4 + 0]);
        if (4 * m4 + 1 > i) acc[4 * m4 + 1] = fmaf(-l.y, q, acc[4 * m4 + 1]);
        if (4 * m4 + 2 > i) acc[4 * m4 + 2] = fmaf(-l.z, q, acc[4 * m4 + 2]);
        if (4 * m4 + 3 > i) acc[4 * m4 + 3] = fmaf(-l.w, q, acc[4 * m4 + 3]);
      }
    }
#pragma unroll
    for (int c = 0; c < KIN; ++c) Out[r * (KIN + 1) + c] = acc[c];
  }
  __syncthreads();
  apply_store(a, blk, r0, nr, Out);
}

__global__ void __launch_bounds__(256) apply2_kernel(ApplyArgs a, ApplyArgs b, int64_t blocks_a) {
  if (blockIdx.x < blocks_a)
    apply_block(a, blockIdx.x);
  else
    apply_block(b, blockIdx.x - blocks_a);
}

// Factor matrices from the sorted eigen-decomposition of the core Gram:
// Mu = W_k (lp x k), Mv = W_k diag(1/sigma) (0 where sigma is negligible),
// S = sigma_k.
__global__ void factor_mats_kernel(const double* eval, const float* evec, int lp, int k, float* Mu, float* Mv,
                                   float* S) {
  // block i, thread j: entry (i, j) of Mu and Mv
  const int i = blockIdx.x, j = threadIdx.x;
  if (j >= k) return;
  const double e0 = eval[0], ev = eval[j];
  const double top = e0 > 0.0 ? sqrt(e0) : 0.0;
  const double sigma = ev > 0.0 ? sqrt(ev) : 0.0;
  const float w = evec[i * lp + j];
  Mu[i * k + j] = w;
  Mv[i * k + j] = (sigma > 1e-12 * top && sigma > 0.0) ? static_cast<float>(w / sigma) : 0.f;
  if (i == 0) S[j] = static_cast<float>(sigma);
}

constexpr int kSignRows = kApplyRows;  // the sign convention's row blocks are the apply kernel's

// One warp per column: lanes take every 32nd block, then a shuffle reduction
// keeps the largest |U| (the lowest block, hence the lowest row, on ties).
__global__ void sign_kernel(const float* __restrict__ U, const float* __restrict__ bmax,
                            const int64_t* __restrict__ bidx, int nblocks, int k, float* sign) {
  const int j = blockIdx.x, lane = threadIdx.x;
  // below every block maximum (colmax reports -1 for a block with no value
  // above -1, e.g. NaN entries), so each lane with a block picks one and the
  // chosen block index is always in range
  float best = -2.f;
  int bb = nblocks;
#pragma unroll 4
  for (int b = lane; b < nblocks; b += 32) {
    const float v = bmax[static_cast<int64_t>(b) * k + j];
    if (v > best) {
      best = v;
      bb = b;
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xFFFFFFFFu, best, o);
    const int ob = __shfl_xor_sync(0xFFFFFFFFu, bb, o);
    if (ov > best || (ov == best && ob < bb)) {
      best = ov;
      bb = ob;
    }
  }
  if (lane == 0) {
    if (bb >= nblocks) bb = 0;   // only when nblocks == 0, which the shape checks exclude
    const int64_t bi = bidx[static_cast<int64_t>(bb) * k + j];
    sign[j] = U[bi * k + j] < 0.f ? -1.f : 1.f;
  }
}


}  // namespace

int64_t apply_blocks(int64_t rows) { return (rows + kApplyRows - 1) / kApplyRows; }

int64_t gram_blocks(int64_t rows) { return (rows + kGramRows - 1) / kGramRows; }

void launch_gram(const float* Y, int64_t rows, int lp, double* gpart, double* G, cudaStream_t s) {
  const int nb = static_cast<int>(gram_blocks(rows));
  const int pairs = (lp / 4) * (lp / 4 + 1) / 2;
  const int threads = (pairs + 31) / 32 * 32;
  gram_kernel<<<nb, threads, kGramRows * (lp + 1) * sizeof(double), s>>>(Y, rows, lp, gpart);
  launch_gram_reduce(gpart, nb, lp, G, s);
}

void launch_gram_reduce(const double* gpart, int nblocks, int lp, double* G, cudaStream_t s) {
  const int nb = lp / 4;
  const int npk = 8 * nb * (nb + 1);
  gram_reduce_kernel<<<(npk + 31) / 32, 32 * kReduceGroups, 0, s>>>(gpart, nblocks, lp, G);
}

bool launch_cholesky(const double* G, int lp, float* Lt, cudaStream_t s) {
  // panels x2, invd, sqd, diag0, L
  const size_t smem = (static_cast<size_t>(lp) * (lp + 1) + 2 * (lp / kTile) * kPanStride + 3 * lp) * sizeof(double);
  if (!ensure_smem(reinterpret_cast<const void*>(cholesky_kernel), smem)) return false;
  cholesky_kernel<<<1, kSmallThreads, smem, s>>>(G, lp, Lt);
  return true;
}

size_t apply_smem(const ApplyArgs& a) {
  return (static_cast<size_t>(a.kin) * a.kout + kApplyRows * (a.kin + 1) + kApplyRows * (a.kout + 1)) *
         sizeof(float);
}

template <int KIN>
bool launch_solve_t(const ApplyArgs& a, cudaStream_t s) {
  const size_t smem = (static_cast<size_t>(KIN) * KIN + 2 * kApplyRows * (KIN + 1)) * sizeof(float);
  if (!ensure_smem(reinterpret_cast<const void*>(solve_kernel<KIN>), smem)) return false;
  solve_kernel<KIN><<<static_cast<unsigned>(apply_blocks(a.rows)), 256, smem, s>>>(a);
  return true;
}

bool launch_solve(const ApplyArgs& a, cudaStream_t s) {
  if (a.kin != a.kout) return false;
  switch (a.kin) {
    case 16: return launch_solve_t<16>(a, s);
    case 32: return launch_solve_t<32>(a, s);
    case 48: return launch_solve_t<48>(a, s);
    case 64: return launch_solve_t<64>(a, s);
    case 80: return launch_solve_t<80>(a, s);
    case 96: return launch_solve_t<96>(a, s);
    case 112: return launch_solve_t<112>(a, s);
    default: return false;
  }
}

void launch_apply(const ApplyArgs& a, cudaStream_t s) {
  const size_t smem = apply_smem(a);
  if (!ensure_smem(reinterpret_cast<const void*>(apply_kernel), smem)) return;
  apply_kernel<<<static_cast<unsigned>(apply_blocks(a.rows)), 256, smem, s>>>(a);
}

void launch_apply2(const ApplyArgs& a, const ApplyArgs& b, cudaStream_t s) {
  const size_t sa = apply_smem(a), sb = apply_smem(b);
  const size_t smem = sa > sb ? sa : sb;
  if (!ensure_smem(reinterpret_cast<const void*>(apply2_kernel), smem)) return;
  const int64_t na = apply_blocks(a.rows), nb = apply_blocks(b.rows);
  apply2_kernel<<<static_cast<unsigned>(na + nb), 256, smem, s>>>(a, b, na);
}

void launch_factor_mats(const double* eval, const float* evec, int lp, int k, float* Mu, float* Mv, float* S,
                        cudaStream_t s) {
  factor_mats_kernel<<<lp, (k + 31) / 32 * 32, 0, s>>>(eval, evec, lp, k, Mu, Mv, S);
}

int64_t sign_blocks(int64_t rows) { return (rows + kSignRows - 1) / kSignRows; }

void launch_signs_from_blocks(float* U, int64_t m, float* V, int64_t n, int k, const float* bmax,
                              const int64_t* bidx, float* sign, cudaStream_t s) {
  (void)V;
  (void)n;
  sign_kernel<<<k, 32, 0, s>>>(U, bmax, bidx, static_cast<int>(sign_blocks(m)), k, sign);
}


}  // namespace metis
