"""Pins of the adaptive spectral learning oracle (oracle/spectral_lr.py,
reading R32): closed-form gains, the identity at cap 1, the scaling of every
kind of component (both sides in the split subspaces, one side, neither),
independence of the sign convention, linearity, the complete-basis case built
entry by entry, and the expanded rank-2k form the library evaluates."""
import numpy as np
import pytest

from oracle import spectral_lr


def _orth(rng, n, k):
    return np.linalg.qr(rng.standard_normal((n, k)))[0]


def _case(seed=0, K=48, N=40, k=6):
    rng = np.random.default_rng(seed)
    U, V = _orth(rng, K, k), _orth(rng, N, k)
    S = np.sort(rng.uniform(0.1, 5.0, k))[::-1]
    G = rng.standard_normal((K, N))
    return rng, U, S, V, G


def test_gains_closed_form():
    S = np.array([4.0, 2.0, 1.0, 0.5])
    assert np.array_equal(spectral_lr.gains(S, 10.0), [1.0, 2.0, 4.0, 8.0])
    assert np.array_equal(spectral_lr.gains(S, 3.0), [1.0, 2.0, 3.0, 3.0])
    assert np.array_equal(spectral_lr.gains([2.0, 0.0], 5.0), [1.0, 1.0])      # a dropped direction
    assert np.array_equal(spectral_lr.gains([0.0, 0.0], 5.0), [1.0, 1.0])
    with pytest.raises(ValueError):
        spectral_lr.gains(S, 0.5)


def test_cap_one_is_the_identity():
    _, U, S, V, G = _case(1)
    assert np.allclose(spectral_lr.scale(G, U, S, V, 1.0), G, rtol=0, atol=1e-13)


def test_components_scale_by_their_gains():
    rng, U, S, V, G = _case(2)
    cap = 6.0
    lam = spectral_lr.gains(S, cap)
    Gs = spectral_lr.scale(G, U, S, V, cap)
    # both sides in the split subspaces: sqrt(lambda_i lambda_j)
    assert np.allclose(U.T @ Gs @ V, np.sqrt(np.outer(lam, lam)) * (U.T @ G @ V), rtol=1e-12, atol=1e-12)
    # one side in the subspace, the other outside: that side's sqrt(lambda)
    w = rng.standard_normal(G.shape[1])
    w -= V @ (V.T @ w)
    z = rng.standard_normal(G.shape[0])
    z -= U @ (U.T @ z)
    assert np.allclose(U.T @ Gs @ w, np.sqrt(lam) * (U.T @ G @ w), rtol=1e-12, atol=1e-12)
    assert np.allclose(z @ Gs @ V, np.sqrt(lam) * (z @ G @ V), rtol=1e-12, atol=1e-12)
    # neither: unchanged (the long tail)
    assert abs(z @ Gs @ w - z @ G @ w) <= 1e-12 * np.linalg.norm(G) * np.linalg.norm(z) * np.linalg.norm(w)
    # the mid and low directions gain, the top one keeps its gradient
    assert lam[0] == 1.0 and np.all(np.diff(lam) >= 0) and lam[-1] > 1.0


def test_sign_convention_and_linearity():
    rng, U, S, V, G = _case(3)
    cap = 4.0
    Gs = spectral_lr.scale(G, U, S, V, cap)
    flip = np.where(rng.random(U.shape[1]) < 0.5, -1.0, 1.0)
    assert np.allclose(spectral_lr.scale(G, U * flip, S, V * flip, cap), Gs, rtol=1e-13, atol=1e-13)
    assert np.allclose(spectral_lr.scale(G, U * flip, S, V, cap), Gs, rtol=1e-13, atol=1e-13)
    H = rng.standard_normal(G.shape)
    lhs = spectral_lr.scale(2.0 * G - 3.0 * H, U, S, V, cap)
    assert np.allclose(lhs, 2.0 * Gs - 3.0 * spectral_lr.scale(H, U, S, V, cap), rtol=1e-12, atol=1e-12)


def test_complete_basis_entry_by_entry():
    # k = K = N: G' = sum_ij sqrt(lambda_i lambda_j) (u_i^T G v_j) u_i v_j^T,
    # assembled one rank-one term at a time
    rng = np.random.default_rng(4)
    n = 7
    U, V = _orth(rng, n, n), _orth(rng, n, n)
    S = np.sort(rng.uniform(0.2, 3.0, n))[::-1]
    G = rng.standard_normal((n, n))
    lam = spectral_lr.gains(S, 100.0)
    want = np.zeros((n, n))
    for i in range(n):
        for j in range(n):
            want += np.sqrt(lam[i] * lam[j]) * (U[:, i] @ G @ V[:, j]) * np.outer(U[:, i], V[:, j])
    assert np.allclose(spectral_lr.scale(G, U, S, V, 100.0), want, rtol=1e-12, atol=1e-12)


def test_expanded_rank_2k_form():
    # G' = G + U a (U^T G) + (G V) a V^T + U a C a V^T, a = sqrt(lambda) - 1, C = U^T G V
    _, U, S, V, G = _case(5)
    a = np.diag(np.sqrt(spectral_lr.gains(S, 5.0)) - 1.0)
    C = U.T @ G @ V
    want = G + U @ a @ (U.T @ G) + (G @ V) @ a @ V.T + U @ a @ C @ a @ V.T
    assert np.allclose(spectral_lr.scale(G, U, S, V, 5.0), want, rtol=1e-12, atol=1e-12)
