"""Randomized spectral split A = U_k diag(S_k) V_k^T + R (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

Sources:
* SII release on Metis, section 2.4 item 1: split the matrix by spectral
  decomposition into a dominant part (largest singular values) and a long-tail
  residual that are quantized independently; use randomized dimension
  reduction so the decomposition runs in a low-dimensional space.
* "Metis: Training LLMs with FP4 Quantization", abstract and technical
  framework: the dominant spectral subspace is preserved under random
  projection and under sparse random sampling, which makes the decomposition
  cost negligible.
* "Metis: Training Large Language Models with Advanced Low-Bit Quantization",
  abstract item (i): spectral decomposition with random embedding separates
  dominant from long-tail components.

The pages give no algorithm; this follows the readings R1-R10 and R22 (sketch
Y = A Omega, subspace iteration re-orthonormalised at every step, core
projection B = Q^T A, SVD of the core, top-k truncation, sign convention,
residual from the unquantized factors).  Everything is float64 numpy/LAPACK.
"""

import numpy as np

from . import sketch


def orth(Y):
    """Orthonormal basis of the column space of Y (Householder QR, LAPACK)."""
    return np.linalg.qr(Y, mode="reduced")[0]


def range_finder(A, omega, power_iters):
    """Q with orthonormal columns spanning (A A^T)^q A Omega, re-orthonormalised
    after every product (reading R2)."""
    Q = orth(A @ omega)
    for _ in range(power_iters):
        Q = orth(A.T @ Q)
        Q = orth(A @ Q)
    return Q


def canonical_signs(U, V):
    """Make each column of U have a positive entry of largest magnitude (the
    lowest row index wins a tie); flip the matching column of V (reading R8)."""
    k = U.shape[1]
    if k == 0:
        return U, V
    idx = np.argmax(np.abs(U), axis=0)
    s = np.sign(U[idx, np.arange(k)])
    s[s == 0] = 1.0
    return U * s, V * s


def core_svd(Q, A, k):
    """SVD of the core B = Q^T A, truncated to the k largest singular values."""
    B = Q.T @ A
    Ub, s, Wt = np.linalg.svd(B, full_matrices=False)
    return Q @ Ub[:, :k], s[:k], Wt[:k].T


def randomized_split(A, k, omega, power_iters):
    """Dominant rank-k factors of A from the sketch Omega (n x l)."""
    A = np.asarray(A, dtype=np.float64)
    Q = range_finder(A, omega, power_iters)
    U, S, V = core_svd(Q, A, k)
    U, V = canonical_signs(U, V)
    return U, S, V


def sampled_split(A, k, omega, rows, power_iters=0):
    """Split using only the sampled rows to find the right singular subspace.

    V_s = top-k right singular vectors of A[rows] (randomized, sketch Omega);
    P = A V_s;  P = Q_P R_P;  R_P = W1 diag(S) W2^T;
    U = Q_P W1,  V = V_s W2, so that U diag(S) V^T = P V_s^T = A V_s V_s^T.
    """
    A = np.asarray(A, dtype=np.float64)
    As = A[rows]
    Q = range_finder(As, omega, power_iters)
    _, _, Vs = core_svd(Q, As, k)
    P = A @ Vs
    Qp, Rp = np.linalg.qr(P, mode="reduced")
    W1, S, W2t = np.linalg.svd(Rp)
    U = Qp @ W1
    V = Vs @ W2t.T
    U, V = canonical_signs(U, V)
    return U, S, V


def residual(A, U, S, V):
    """R = A - U diag(S) V^T (float64, from the unquantized factors, R10)."""
    return np.asarray(A, dtype=np.float64) - (U * S) @ V.T


def compensated_residual(A, Uq, S, Vq):
    """R = A - deq(U_q) diag(S) deq(V_q)^T (float64): the residual against
    the FP4 factors as quantized (the variant of R10 that the option
    `compensate` selects; reading R29).  Uq, Vq: FP4Tensor with outer = k
    (inner m and n)."""
    Ud = Uq.dequantize().T          # m x k
    Vd = Vq.dequantize().T          # n x k
    return np.asarray(A, dtype=np.float64) - (Ud * np.asarray(S, dtype=np.float64)) @ Vd.T


def make_sketch(n, l, seed, kind="gaussian", nnz=4):
    if kind == "gaussian":
        return sketch.gaussian_omega(n, l, seed)
    if kind == "sparse_sign":
        return sketch.sparse_sign_omega(n, l, nnz, seed)
    raise ValueError(kind)


def split(A, k, p, power_iters, seed, kind="gaussian", nnz=4, sample_rows=0):
    """Full split of A (m x n) as the library computes it.

    Returns dict(U, S, V, R, omega, rows)."""
    A = np.asarray(A, dtype=np.float64)
    m, n = A.shape
    l = k + p
    omega = make_sketch(n, l, seed, kind, nnz)
    rows = None
    if sample_rows:
        rows = sketch.sample_rows(m, sample_rows, seed)
        U, S, V = sampled_split(A, k, omega, rows, power_iters)
    else:
        U, S, V = randomized_split(A, k, omega, power_iters)
    return dict(U=U, S=S, V=V, R=residual(A, U, S, V), omega=omega, rows=rows)
