"""Pins for the oracle's W4A4G4 MLP training step (reading R31): the float64
gradients against finite differences, the FP4 products' quantization axes and
operand roles (exact on operands every axis represents exactly), the metis
operands reassembling the weight, and training under every policy."""
import warnings

import numpy as np
import pytest

from oracle import fp4, gemm, mlp


def _rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def test_exact_gradients_match_finite_differences():
    X, T, (W1, W2) = mlp.problem(n=6, d_in=5, d_h=7, d_out=3, seed=1)
    pol = mlp.Policy("exact")
    _, (g1, g2) = mlp.loss_and_grads((W1, W2), X, T, pol)
    h = 1e-6
    for g, which in ((g1, 0), (g2, 1)):
        num = np.zeros_like(g)
        for idx in np.ndindex(g.shape):
            P = [W1.copy(), W2.copy()]
            P[which][idx] += h
            lp, _ = mlp.loss_and_grads(tuple(P), X, T, pol)
            P[which][idx] -= 2 * h
            lm, _ = mlp.loss_and_grads(tuple(P), X, T, pol)
            num[idx] = (lp - lm) / (2 * h)
        assert np.max(np.abs(num - g)) <= 1e-6 * max(1.0, np.max(np.abs(g)))


def _representable(shape, seed):
    # E2M1 values at one power of two: every block along either axis holds
    # them exactly in MXFP4 (the block scale only moves to a smaller power)
    rng = np.random.default_rng(seed)
    vals = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    x = rng.choice(vals, size=shape) * rng.choice([-1, 1], size=shape)
    return x * 2.0 ** -3


def test_fp4_products_exact_on_representable_operands():
    X, W, dZ = _representable((64, 96), 1), _representable((96, 32), 2), _representable((64, 32), 3)
    for x in (X, W, dZ):                  # the premise: both axes are exact
        for axis in (0, 1):
            assert np.array_equal(fp4.quantize(np.float32(x), "mx", axis).dequantize() if axis == 1 else
                                  fp4.quantize(np.float32(x), "mx", axis).dequantize().T, x)
    pol = mlp.Policy("fp4", "mx")
    assert np.array_equal(mlp.forward(X, W, pol), X @ W)
    dX, dW = mlp.backward(dZ, X, W, pol)
    assert np.array_equal(dX, dZ @ W.T) and np.array_equal(dW, X.T @ dZ)


def test_metis_operands_reassemble_the_weight():
    rng = np.random.default_rng(4)
    K, N = 128, 96
    U, _ = np.linalg.qr(rng.standard_normal((K, K)))
    V, _ = np.linalg.qr(rng.standard_normal((N, N)))
    s = np.concatenate([[40, 20, 10, 5], 0.1 * np.ones(N - 4)])
    W = (U[:, :N] * s) @ V.T
    pol = mlp.Policy("metis", "nv", k=8, p=8, q=1, seed=2)
    sp = mlp._split(W, pol, 0)
    q = lambda a, ax: fp4.quantize(np.float32(a), "nv", ax)
    fwd = gemm.Operand(q(sp["R"], 0), 8, q(sp["U"], 0), q(sp["V"], 0), sp["S"])     # W: K x N
    bwd = gemm.Operand(q(sp["R"], 1), 8, q(sp["V"], 0), q(sp["U"], 0), sp["S"])     # W^T: N x K
    # FP4 error of the factors (the dominant energy) is about 0.13 here; a
    # swapped role or axis gives a shape error or an error near 1
    assert _rel(gemm.dense_right(fwd), W) < 0.2
    assert _rel(gemm.dense_right(bwd), W.T) < 0.2
    # the products the policy forms are these operands' products
    X = rng.standard_normal((64, K))
    dZ = rng.standard_normal((64, N))
    assert _rel(mlp.forward(X, W, pol), X @ W) < 0.3
    dX, dW = mlp.backward(dZ, X, W, pol)
    assert _rel(dX, dZ @ W.T) < 0.3 and _rel(dW, X.T @ dZ) < 0.3


@pytest.mark.parametrize("fmt", ["nv", "mx"])
def test_every_policy_trains(fmt):
    warnings.simplefilter("ignore", RuntimeWarning)
    X, T, params = mlp.problem(n=128, d_in=64, d_h=64, d_out=32, seed=0)
    final = {}
    for kind in ("exact", "fp4", "metis"):
        losses, _ = mlp.train(params, X, T, mlp.Policy(kind, fmt, k=8, p=8, q=1, seed=1), lr=1.0, steps=30)
        assert np.all(np.isfinite(losses))
        assert losses[-1] < 0.5 * losses[0]
        final[kind] = losses[-1]
    assert np.all(np.diff(mlp.train(params, X, T, mlp.Policy("exact"), lr=1.0, steps=30)[0]) < 0)
    for kind in ("fp4", "metis"):
        assert final[kind] < 1.5 * final["exact"]
