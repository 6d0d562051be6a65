"""A small synthetic MLP trained with W4A4G4 linear layers (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

Sources: "Metis: Training LLMs with FP4 Quantization" abstract (W4A4G4:
weights, activations and gradients in FP4 in the forward and both backward
products; the split keeps the FP4 training loss close to the higher-precision
run); SII release section 2.4 item 1 (the dominant low-rank part and the
long-tail residual are quantized independently).

Reading R31 (the training workload): a two-layer ReLU regression
Y = relu(X W1) W2 with loss L = ||Y - T||^2 / (2 n d_out), trained by plain SGD.
Every linear layer Z = X W runs its three products under one precision
policy:

  "exact"  float64 products;
  "fp4"    FP4 operands, each quantized along the product's contraction axis
           (forward: X and W along K; dX = dZ W^T: dZ and W along N;
           dW = X^T dZ: X and dZ along M);
  "metis"  as "fp4", but the weight and the output gradient enter as spectral
           split operands R_q + U_q diag(S) V_q^T (the oracle's split, R
           quantized along the contraction axis, U_q and V_q along their long
           axis), the operand roles of the library's linear products
           (forward: P = U_W, F = V_W; dX: P = V_W, F = U_W; dW: P = U_dZ,
           F = V_dZ).
The activation function, loss and update run in float64.  The float32 values
that get quantized are fl32 of the float64 ones.
"""

import numpy as np

from . import fp4, gemm
from . import split as spectral


class Policy:
    def __init__(self, kind="exact", fmt="nv", k=8, p=8, q=1, seed=0):
        if kind not in ("exact", "fp4", "metis"):
            raise ValueError("policy is exact, fp4 or metis")
        self.kind, self.fmt, self.k, self.p, self.q, self.seed = kind, fmt, k, p, q, seed


def _q(x, fmt, axis):
    return fp4.quantize(np.float32(x), fmt, axis)


def _split(A, pol, salt):
    s = spectral.split(A, pol.k, pol.p, pol.q, pol.seed + salt)
    return s


def forward(X, W, pol, salt=0):
    """Z = X W under the policy (X: n x K, W: K x N)."""
    if pol.kind == "exact":
        return X @ W
    left = gemm.Operand(_q(X, pol.fmt, 1))                      # X along K
    if pol.kind == "fp4":
        right = gemm.Operand(_q(W, pol.fmt, 0))                 # W along K
    else:
        s = _split(W, pol, salt)
        right = gemm.Operand(_q(s["R"], pol.fmt, 0), pol.k, _q(s["U"], pol.fmt, 0), _q(s["V"], pol.fmt, 0),
                             s["S"])
    return gemm.gemm(left, right)


def backward(dZ, X, W, pol, salt=0, need_dx=True):
    """(dX, dW) of Z = X W under the policy: dX = dZ W^T, dW = X^T dZ."""
    if pol.kind == "exact":
        return (dZ @ W.T if need_dx else None), X.T @ dZ
    fmt = pol.fmt
    sd = _split(dZ, pol, salt + 1) if pol.kind == "metis" else None
    sw = _split(W, pol, salt) if (pol.kind == "metis" and need_dx) else None
    dX = None
    if need_dx:
        # contraction over N: dZ along N (left), W^T along N (right, stored K x N rows)
        if sd is None:
            left = gemm.Operand(_q(dZ, fmt, 1))
        else:
            left = gemm.Operand(_q(sd["R"], fmt, 1), pol.k, _q(sd["V"], fmt, 0), _q(sd["U"], fmt, 0), sd["S"])
        if sw is None:
            right = gemm.Operand(_q(W, fmt, 1))
        else:
            right = gemm.Operand(_q(sw["R"], fmt, 1), pol.k, _q(sw["V"], fmt, 0), _q(sw["U"], fmt, 0), sw["S"])
        dX = gemm.gemm(left, right)
    # contraction over M (the batch): X^T along M (left), dZ along M (right)
    left = gemm.Operand(_q(X, fmt, 0))
    if sd is None:
        right = gemm.Operand(_q(dZ, fmt, 0))
    else:
        right = gemm.Operand(_q(sd["R"], fmt, 0), pol.k, _q(sd["U"], fmt, 0), _q(sd["V"], fmt, 0), sd["S"])
    return dX, gemm.gemm(left, right)


def loss_and_grads(params, X, T, pol, step=0):
    """Loss and (dW1, dW2) of the two-layer regression at ``params``."""
    W1, W2 = params
    n = X.shape[0]
    Z1 = forward(X, W1, pol, salt=8 * step)
    A1 = np.maximum(Z1, 0.0)
    Y = forward(A1, W2, pol, salt=8 * step + 2)
    D = Y - T
    loss = 0.5 * float(np.sum(D * D)) / D.size
    dY = D / D.size
    dA1, dW2 = backward(dY, A1, W2, pol, salt=8 * step + 4)
    dZ1 = dA1 * (Z1 > 0)
    _, dW1 = backward(dZ1, X, W1, pol, salt=8 * step + 6, need_dx=False)
    return loss, (dW1, dW2)


def train(params, X, T, pol, lr, steps):
    """Plain SGD; returns the loss before every step and the final params."""
    losses = []
    W1, W2 = params
    for t in range(steps):
        loss, (dW1, dW2) = loss_and_grads((W1, W2), X, T, pol, step=t)
        losses.append(loss)
        W1, W2 = W1 - lr * dW1, W2 - lr * dW2
    return np.array(losses), (W1, W2)


def problem(n=256, d_in=128, d_h=128, d_out=64, seed=0):
    """Teacher-student data with anisotropic spectra: inputs with a decaying
    covariance spectrum, a teacher of the same architecture whose weights
    have decaying singular values, and a student initialised at small
    random weights.  Returns X, T, (W1, W2)."""
    rng = np.random.default_rng(seed)

    def decaying(rows, cols, rate):
        Ua, _ = np.linalg.qr(rng.standard_normal((rows, min(rows, cols))))
        Va, _ = np.linalg.qr(rng.standard_normal((cols, min(rows, cols))))
        s = 1.0 / (1.0 + np.arange(min(rows, cols))) ** rate
        return (Ua * s) @ Va.T

    Dx = decaying(d_in, d_in, 0.5)
    X = rng.standard_normal((n, d_in)) @ Dx * np.sqrt(d_in / np.sum(Dx * Dx))   # E x_ij^2 = 1
    A1, A2 = decaying(d_in, d_h, 1.0) * 4.0, decaying(d_h, d_out, 1.0) * 4.0
    T = np.maximum(X @ A1, 0.0) @ A2
    T = T / np.std(T)                      # unit-variance targets
    W1 = rng.standard_normal((d_in, d_h)) / np.sqrt(d_in)
    W2 = rng.standard_normal((d_h, d_out)) / np.sqrt(d_h)
    return X, T, (W1, W2)
