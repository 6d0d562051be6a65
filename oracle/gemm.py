"""W4A4G4 split-linear GEMMs on FP4 operands (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

Sources: "Metis: Training LLMs with FP4 Quantization", abstract (W4A4G4:
weights, activations and gradients in FP4 for the forward and both backward
products); SII release section 2.4 item 1 (dominant and long-tail parts are
quantized independently and both take part in the product); retelling of
arXiv 2603.10444, Averis paragraphs (the output combines the quantized mean and
the quantized residual; the split keeps the product mathematically equivalent
before quantization).

An operand of C = A B is a sum of a quantized residual and an optional
low-rank term (readings R14-R17):

    left  operand  A (M x K) = R_A + F_A diag(S_A) P_A^T
    right operand  B (K x N) = R_B + P_B diag(S_B) F_B^T

R is stored quantized along the contraction axis K (outer = M for A, N for B).
P (K x k) is the factor that runs along the contraction axis and F (M x k or
N x k) the one along the free axis; both are stored quantized along their long
axis (outer = k).  A factor may instead be the all-ones vector (the Averis
mean split, where k = 1).  The oracle's product is the plain float64 product
of the two dequantized dense operands.
"""

import numpy as np


class Operand:
    """Oracle-side operand: R (FP4Tensor), optional k, P, F (FP4Tensor or the
    string "ones") and S (float array)."""

    def __init__(self, R, k=0, P=None, F=None, S=None):
        self.R = R
        self.k = k
        self.P = P
        self.F = F
        self.S = None if S is None else np.asarray(S, dtype=np.float64)


def _factor(f, length, k):
    if isinstance(f, str) and f == "ones":
        return np.ones((length, k))
    d = f.dequantize()              # k x length
    if d.shape != (k, length):
        raise ValueError("factor has the wrong shape")
    return d.T


def dense_left(op):
    """Dense M x K float64 value of a left operand."""
    A = op.R.dequantize()           # M x K
    if op.k:
        M, K = A.shape
        A = A + (_factor(op.F, M, op.k) * op.S) @ _factor(op.P, K, op.k).T
    return A


def dense_right(op):
    """Dense K x N float64 value of a right operand."""
    B = op.R.dequantize().T         # stored N x K
    if op.k:
        K, N = B.shape
        B = B + (_factor(op.P, K, op.k) * op.S) @ _factor(op.F, N, op.k).T
    return B


def gemm(opA, opB, rows=None):
    """C = dense(A) @ dense(B) in float64; ``rows`` restricts to those output
    rows (rows are independent, so the subset is exact)."""
    A = dense_left(opA)
    if rows is not None:
        A = A[rows]
    return A @ dense_right(opB)
