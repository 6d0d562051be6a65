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

from . import fp4


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


# ---------------------------------------------------------------------------
# Re-quantized low-rank intermediates (reading R30)
# ---------------------------------------------------------------------------

def intermediates(opA, opB):
    """The low-rank intermediates of C = A B in float64 (reading R16):

        C = R_A R_B + T1 F_B^T + F_A T2,
        T1 = (R_A P_B + F_A diag(S_A) P_A^T P_B) diag(S_B)   (M x k_B),
        T2 = diag(S_A) P_A^T R_B                             (k_A x N).

    Returns (R_A, R_B, T1, F_B, F_A, T2); the absent terms are None."""
    RA = opA.R.dequantize()                     # M x K
    RB = opB.R.dequantize().T                   # K x N
    M, K = RA.shape
    N = RB.shape[1]
    FA = PA = FB = PB = T1 = T2 = None
    if opA.k:
        FA = _factor(opA.F, M, opA.k)           # M x k_A
        PA = _factor(opA.P, K, opA.k)           # K x k_A
        T2 = (PA * opA.S).T @ RB
    if opB.k:
        PB = _factor(opB.P, K, opB.k)           # K x k_B
        FB = _factor(opB.F, N, opB.k)           # N x k_B
        T1 = RA @ PB
        if opA.k:
            T1 = T1 + (FA * opA.S) @ (PA.T @ PB)
        T1 = T1 * opB.S
    return RA, RB, T1, FB, FA, T2


def requantize(X32, fmt, axis):
    """deq(Q(X)) for a float32 matrix, blocks along ``axis`` (1: along the
    columns, 0: along the rows).  A blocked length that is not a multiple of
    the block size is zero-padded to one; the zeros change no block maximum
    and are dropped again (reading R30)."""
    X32 = np.asarray(X32, dtype=np.float32)
    bs = 32 if fmt == "mx" else 16
    n = X32.shape[axis]
    pad = (-n) % bs
    if pad:
        widths = [(0, 0), (0, 0)]
        widths[axis] = (0, pad)
        X32 = np.pad(X32, widths)
    d = fp4.quantize(X32, fmt, axis).dequantize()      # outer x inner
    if axis == 0:
        d = d.T
    return d[:, :n] if axis == 1 else d[:n, :]


def gemm_requant(opA, opB, fmt, t1_32=None, t2_32=None):
    """C = A B with the low-rank intermediates re-quantized to FP4 along the
    axis they are contracted over (reading R30): T1 (M x k_B) in blocks along
    k_B, T2 (k_A x N) in blocks along k_A, each with its own NVFP4 tensor
    scale.  The values quantized are float32: by default fl32 of the exact
    T1 / T2; ``t1_32`` / ``t2_32`` supply other float32 values (the ones a
    device computed), so that both sides take the same FP4 decisions.  The
    factors F_A, F_B enter as they are (already FP4)."""
    RA, RB, T1, FB, FA, T2 = intermediates(opA, opB)
    C = RA @ RB
    if T1 is not None:
        v = np.float32(T1) if t1_32 is None else np.asarray(t1_32, dtype=np.float32)
        C = C + requantize(v, fmt, 1) @ FB.T
    if T2 is not None:
        v = np.float32(T2) if t2_32 is None else np.asarray(t2_32, dtype=np.float32)
        C = C + FA @ requantize(v, fmt, 0)
    return C
