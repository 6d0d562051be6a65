"""A small synthetic MLP trained with W4A4G4 linear layers on the GPU.

Source: "Metis: Training LLMs with FP4 Quantization" abstract (W4A4G4: the
forward product and both backward products of every linear layer run on FP4
operands, and the spectral split keeps the FP4 training loss close to the
higher-precision run); SII release section 2.4 item 1 (the dominant low-rank
part and the long-tail residual are quantized independently).

The workload (reading R31): a two-layer ReLU regression Y = relu(X W1) W2 with
loss ||Y - T||^2 / (2 n d_out), trained by plain SGD.  Every product of every
layer goes through the library's C ABI under one policy:

  "fp4"    each operand quantized along the product's contraction axis
           (forward: X and W along K; dX = dZ W^T: dZ and W along N;
           dW = X^T dZ: X and dZ along M);
  "metis"  as "fp4", but the weight and the output gradient enter as spectral
           split operands (metis_split: R_q + U_q diag(S) V_q^T), in the
           operand roles of metis_linear_fwd / metis_linear_bwd.

The products, quantizations and splits all run in the library's kernels; the
ReLU, its mask, the loss and the SGD update are the workload around the layer
and run as float32 torch operations.  ``step`` returns every product's FP4
operands and output, so that a test can hold each product to the oracle's
float64 product of exactly those operands.
"""
import torch

from . import api


class Policy:
    def __init__(self, kind="fp4", fmt="nv", k=8, p=8, q=1, seed=0):
        if kind not in ("fp4", "metis"):
            raise ValueError("policy is fp4 or metis")
        self.kind, self.fmt, self.k, self.p, self.q, self.seed = kind, fmt, k, p, q, seed


def _split(A, pol, salt):
    return api.split(A.contiguous(), pol.k, pol.p, pol.q, pol.seed + salt, pol.fmt, rows=True, cols=True)


def forward(X, W, pol, salt, record):
    """Z = X W (X: n x K, W: K x N, float32 CUDA tensors)."""
    M, K = X.shape
    N = W.shape[1]
    xop = api.Operand(api.quantize_fp4(X.contiguous(), pol.fmt, 1))          # X along K
    if pol.kind == "fp4":
        wop = api.Operand(api.quantize_fp4(W.contiguous(), pol.fmt, 0))      # W along K
    else:
        wop = _split(W, pol, salt).operand("right")
    Z = api.linear_fwd(xop, wop, M, N, K)
    record.append(("fwd", xop, wop, Z))
    return Z


def backward(dZ, X, W, pol, salt, record, need_dx=True):
    """(dX, dW) of Z = X W: dX = dZ W^T (contraction over N), dW = X^T dZ
    (contraction over the batch M)."""
    M, K = X.shape
    N = W.shape[1]
    if pol.kind == "fp4":
        dz_n = api.Operand(api.quantize_fp4(dZ.contiguous(), pol.fmt, 1))    # dZ along N
        dz_m = api.Operand(api.quantize_fp4(dZ.contiguous(), pol.fmt, 0))    # dZ along M
        wt = api.Operand(api.quantize_fp4(W.contiguous(), pol.fmt, 1)) if need_dx else None   # W^T along N
    else:
        sd = _split(dZ, pol, salt + 1)
        dz_n, dz_m = sd.operand("left"), sd.operand("right")
        wt = None
        if need_dx:
            sw = _split(W, pol, salt)
            wt = api.Operand(sw.R_rows, pol.k, sw.V_q, sw.U_q, sw.S)
    xt = api.Operand(api.quantize_fp4(X.contiguous(), pol.fmt, 0))           # X^T along M
    dX, dW = api.linear_bwd(dz_n if need_dx else None, wt, xt, dz_m, M, N, K, want_dx=need_dx)
    if need_dx:
        record.append(("dx", dz_n, wt, dX))
    record.append(("dw", xt, dz_m, dW))
    return dX, dW


def step(params, X, T, pol, t=0):
    """Loss and (dW1, dW2) at ``params``; also the record of every product:
    (name, left operand, right operand, output)."""
    W1, W2 = params
    record = []
    Z1 = forward(X, W1, pol, 8 * t, record)
    A1 = torch.relu(Z1)
    Y = forward(A1, W2, pol, 8 * t + 2, record)
    D = Y - T
    loss = 0.5 * float((D * D).sum()) / D.numel()
    dY = D / D.numel()
    dA1, dW2 = backward(dY, A1, W2, pol, 8 * t + 4, record)
    dZ1 = dA1 * (Z1 > 0)
    _, dW1 = backward(dZ1, X, W1, pol, 8 * t + 6, record, need_dx=False)
    return loss, (dW1, dW2), record


def train(params, X, T, pol, lr, steps):
    """Plain SGD; returns the loss before every step and the final params."""
    W1, W2 = params
    losses = []
    for t in range(steps):
        loss, (dW1, dW2), _ = step((W1, W2), X, T, pol, t)
        losses.append(loss)
        W1, W2 = W1 - lr * dW1, W2 - lr * dW2
    return losses, (W1, W2)
