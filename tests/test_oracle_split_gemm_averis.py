"""Pins for the oracle's randomized split, split-operand GEMM and Averis split:
exact-rank recovery, the Eckart-Young tail, projector identities, brute-force
exact products, the four-term expansion of a split x split product, and the
mean/residual reconstruction."""
from fractions import Fraction

import numpy as np
import pytest

from oracle import averis, fp4, gemm, sketch, split


def _rng(s):
    return np.random.default_rng(s)


# --------------------------------------------------------------------------
# split
# --------------------------------------------------------------------------

@pytest.mark.parametrize("q", [0, 1, 2])
def test_exact_rank_recovered(q):
    rng = _rng(1)
    m, n, r, k, p = 200, 150, 6, 8, 8
    A = rng.standard_normal((m, r)) @ rng.standard_normal((r, n))
    om = sketch.gaussian_omega(n, k + p, 3)
    U, S, V = split.randomized_split(A, k, om, q)
    R = split.residual(A, U, S, V)
    assert np.linalg.norm(R) / np.linalg.norm(A) < 1e-12


def test_eckart_young_tail_full_sketch():
    # with l = n the sketch spans everything: R is the optimal rank-k residual
    rng = _rng(2)
    m, n, k = 60, 40, 7
    A = rng.standard_normal((m, n)) * np.exp(-0.15 * np.arange(n))
    om = sketch.gaussian_omega(n, n, 4)
    U, S, V = split.randomized_split(A, k, om, 0)
    sv = np.linalg.svd(A, compute_uv=False)
    R = split.residual(A, U, S, V)
    assert abs(np.sum(R ** 2) - np.sum(sv[k:] ** 2)) <= 1e-10 * np.sum(sv ** 2)
    assert np.allclose(S, sv[:k], rtol=1e-12)


def test_rank_at_most_l_is_exact_tail():
    rng = _rng(3)
    m, n, k, p = 80, 70, 5, 5
    A = rng.standard_normal((m, k + p)) @ rng.standard_normal((k + p, n))
    om = sketch.gaussian_omega(n, k + p, 5)
    U, S, V = split.randomized_split(A, k, om, 0)
    sv = np.linalg.svd(A, compute_uv=False)
    R = split.residual(A, U, S, V)
    assert abs(np.sum(R ** 2) - np.sum(sv[k:] ** 2)) <= 1e-9 * np.sum(sv ** 2)


def test_factor_invariants_and_sign_convention():
    rng = _rng(4)
    m, n, k, p = 300, 200, 12, 8
    A = rng.standard_normal((m, n)) + 5 * np.outer(rng.standard_normal(m), rng.standard_normal(n)) / 10
    om = sketch.gaussian_omega(n, k + p, 6)
    U, S, V = split.randomized_split(A, k, om, 1)
    R = split.residual(A, U, S, V)
    assert np.allclose(U.T @ U, np.eye(k), atol=1e-12)
    assert np.allclose(V.T @ V, np.eye(k), atol=1e-12)
    assert np.all(np.diff(S) <= 0) and np.all(S >= 0)
    # U_k^T R = 0 holds exactly for the randomized split (U_k^T A = S_k V_k^T)
    assert np.linalg.norm(U.T @ R) < 1e-12 * np.linalg.norm(A)
    idx = np.argmax(np.abs(U), axis=0)
    assert np.all(U[idx, np.arange(k)] > 0)


def test_power_iteration_spans_krylov_product():
    # re-orthonormalised subspace iteration spans (A A^T)^q A Omega
    rng = _rng(5)
    m, n, l = 50, 40, 6
    A = rng.standard_normal((m, n))
    om = sketch.gaussian_omega(n, l, 7)
    Q = split.range_finder(A, om, 2)
    Y = A @ A.T @ A @ A.T @ A @ om
    Qy = np.linalg.svd(Y, full_matrices=False)[0]
    assert np.allclose(Q @ Q.T, Qy @ Qy.T, atol=1e-9)


def test_halko_martinsson_tropp_range():
    # average-case bound (HMT 2011, Thm 10.5 with q = 0):
    # E||A - QQ^T A||_F <= (1 + k/(p-1))^(1/2) (sum_{j>k} s_j^2)^(1/2)
    rng = _rng(6)
    m, n, k, p = 120, 100, 10, 6
    A = rng.standard_normal((m, n)) * np.exp(-0.05 * np.arange(n))
    sv = np.linalg.svd(A, compute_uv=False)
    bound = np.sqrt(1 + k / (p - 1)) * np.sqrt(np.sum(sv[k:] ** 2))
    errs = []
    for s in range(20):
        Q = split.range_finder(A, sketch.gaussian_omega(n, k + p, 100 + s), 0)
        errs.append(np.linalg.norm(A - Q @ (Q.T @ A)))
    assert np.mean(errs) <= 1.1 * bound
    assert np.min(errs) >= np.sqrt(np.sum(sv[k + p:] ** 2)) * (1 - 1e-9)


def test_sampled_split_identities():
    rng = _rng(7)
    m, n, k, p = 400, 64, 6, 6
    A = rng.standard_normal((m, n)) + 8 * np.outer(rng.standard_normal(m), rng.standard_normal(n)) / 8
    om = sketch.sparse_sign_omega(n, k + p, 4, 9)
    rows = sketch.sample_rows(m, 100, 9)
    U, S, V = split.sampled_split(A, k, om, rows)
    R = split.residual(A, U, S, V)
    # the dominant part is the projection of A onto span(V_s) = span(V)
    assert np.allclose(R, A - A @ V @ V.T, atol=1e-10)
    assert np.allclose(U.T @ U, np.eye(k), atol=1e-12)
    assert np.allclose(V.T @ V, np.eye(k), atol=1e-12)
    # with all rows sampled and a full sketch the split is the truncated SVD
    om_full = sketch.gaussian_omega(n, n, 10)
    U2, S2, V2 = split.sampled_split(A, k, om_full, np.arange(m))
    sv = np.linalg.svd(A, compute_uv=False)
    assert np.allclose(S2, sv[:k], rtol=1e-10)


def test_split_driver_shapes():
    rng = _rng(8)
    A = rng.standard_normal((64, 48))
    out = split.split(A, 4, 4, 1, 0)
    assert out["U"].shape == (64, 4) and out["V"].shape == (48, 4) and out["R"].shape == (64, 48)
    out = split.split(A, 4, 4, 0, 0, kind="sparse_sign", nnz=2, sample_rows=20)
    assert out["rows"].shape == (20,)


# --------------------------------------------------------------------------
# GEMM
# --------------------------------------------------------------------------

def _q(X, fmt, axis=1):
    return fp4.quantize(np.asarray(X, np.float32), fmt, axis)


@pytest.mark.parametrize("fmt", ["mx", "nv"])
def test_gemm_matches_exact_rational_product(fmt):
    rng = _rng(10)
    M, N, K = 5, 4, 64
    A = _q(rng.standard_normal((M, K)) * 3, fmt)
    B = _q(rng.standard_normal((N, K)), fmt)          # stored N x K (right operand)
    C = gemm.gemm(gemm.Operand(A), gemm.Operand(B))
    Ad, Bd = A.dequantize(), B.dequantize()
    for i in range(M):
        for j in range(N):
            terms = [Fraction(Ad[i, t]) * Fraction(Bd[j, t]) for t in range(K)]
            exact = sum(terms)
            if fmt == "mx":
                # dyadic values with a narrow exponent range: the float64 sum is exact
                assert Fraction(C[i, j]) == exact
            else:
                # float64 dot-product bound: K u sum |a_t b_t|
                assert abs(Fraction(C[i, j]) - exact) <= K * Fraction(1, 2 ** 53) * sum(abs(t) for t in terms)


def test_split_operand_four_term_expansion():
    # A B = R_A R_B + T1 F_B^T + F_A T2 with
    # T1 = (R_A P_B + F_A S_A (P_A^T P_B)) S_B and T2 = S_A P_A^T R_B
    rng = _rng(11)
    M, N, K, ka, kb = 48, 64, 96, 3, 5
    fmt = "nv"
    RA, RB = _q(rng.standard_normal((M, K)), fmt), _q(rng.standard_normal((N, K)), fmt)
    PA, FA = _q(rng.standard_normal((ka, K)), fmt), _q(rng.standard_normal((ka, M)), fmt)
    PB, FB = _q(rng.standard_normal((kb, K)), fmt), _q(rng.standard_normal((kb, N)), fmt)
    SA, SB = rng.random(ka) + 1, rng.random(kb) + 1
    C = gemm.gemm(gemm.Operand(RA, ka, PA, FA, SA), gemm.Operand(RB, kb, PB, FB, SB))
    rA, rB = RA.dequantize(), RB.dequantize().T
    pA, fA, pB, fB = PA.dequantize().T, FA.dequantize().T, PB.dequantize().T, FB.dequantize().T
    T1 = (rA @ pB + (fA * SA) @ (pA.T @ pB)) * SB
    T2 = SA[:, None] * (pA.T @ rB)
    C2 = rA @ rB + T1 @ fB.T + fA @ T2
    assert np.allclose(C, C2, rtol=1e-12, atol=1e-12 * np.abs(C).max())


def test_averis_operand_rank_one():
    rng = _rng(12)
    M, N, K = 32, 16, 64
    RA = _q(rng.standard_normal((M, K)), "nv")
    mu = _q(rng.standard_normal((1, K)) * 5, "nv")
    RB = _q(rng.standard_normal((N, K)), "nv")
    C = gemm.gemm(gemm.Operand(RA, 1, P=mu, F="ones", S=[1.0]), gemm.Operand(RB))
    want = RA.dequantize() @ RB.dequantize().T + (mu.dequantize() @ RB.dequantize().T)
    assert np.allclose(C, want, rtol=1e-12, atol=1e-12)


def test_gemm_row_subset():
    rng = _rng(13)
    A = _q(rng.standard_normal((64, 64)), "mx")
    B = _q(rng.standard_normal((32, 64)), "mx")
    full = gemm.gemm(gemm.Operand(A), gemm.Operand(B))
    rows = np.array([0, 7, 63])
    assert np.array_equal(gemm.gemm(gemm.Operand(A), gemm.Operand(B), rows=rows), full[rows])


# --------------------------------------------------------------------------
# Averis
# --------------------------------------------------------------------------

def test_averis_reconstruction_and_zero_column_sums():
    rng = _rng(14)
    X = rng.standard_normal((500, 64)) * 3 + rng.standard_normal(64) * 5
    mu, R = averis.split(X)
    rec = R + mu[None, :]
    # two roundings, each at most half an ulp of the largest magnitude involved
    big = np.maximum(np.maximum(np.abs(X), np.abs(R)), np.abs(mu)[None, :])
    assert np.all(np.abs(rec - X) <= np.spacing(big))
    assert np.all(np.abs(R.sum(axis=0)) < 1e-9 * np.abs(X).sum(axis=0))


def test_averis_pure_mean():
    mu0 = np.linspace(-3, 5, 33)
    X = np.tile(mu0, (2 ** 15, 1))
    mu, R = averis.split(X)
    assert np.array_equal(mu, mu0)
    assert np.all(R == 0)


def test_averis_residual_amax_from_columns():
    rng = _rng(15)
    X = (rng.standard_normal((300, 40)) * 4).astype(np.float32)
    mu = X.astype(np.float64).mean(axis=0).astype(np.float32)
    r = averis.residual_f32(X, mu)
    assert averis.residual_amax_from_columns(X, mu) == np.abs(r).max()


# --------------------------------------------------------------------------
# error-compensated residual (R29)
# --------------------------------------------------------------------------

def test_compensated_residual_equals_plain_for_representable_factors():
    # factors whose entries are FP4 values times a power-of-two block scale
    # are exact in MXFP4: the compensated residual is the plain one
    rng = _rng(41)
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    U = rng.choice(grid, (64, 4)) * rng.choice([-1.0, 1.0], (64, 4)) / 8.0
    V = rng.choice(grid, (96, 4)) * rng.choice([-1.0, 1.0], (96, 4)) / 16.0
    U[0] = 6.0 / 8.0          # every 32-row block keeps its maximum at 6 x scale
    U[32] = 6.0 / 8.0
    V[0] = V[32] = V[64] = 6.0 / 16.0
    S = np.array([3.0, 2.0, 1.5, 1.0])
    A = rng.standard_normal((64, 96))
    Uq = fp4.quantize(U.astype(np.float32), "mx", 0)
    Vq = fp4.quantize(V.astype(np.float32), "mx", 0)
    assert np.array_equal(Uq.dequantize().T, U) and np.array_equal(Vq.dequantize().T, V)
    assert np.array_equal(split.compensated_residual(A, Uq, S, Vq), split.residual(A, U, S, V))


@pytest.mark.parametrize("fmt", ["nv", "mx"])
def test_compensated_residual_absorbs_the_factor_error(fmt):
    # with an exact (unquantized) residual the compensated operand is A
    # itself, while the plain residual leaves the factors' FP4 error; after
    # quantizing the residual too, the compensated operand is the closer one
    rng = _rng(42)
    m, n, k = 256, 192, 16
    A = (rng.standard_normal((m, k)) * (8.0 / (1 + np.arange(k)))) @ rng.standard_normal((k, n)) / np.sqrt(n)
    A += 0.02 * rng.standard_normal((m, n))
    r = split.split(A, k, 8, 1, 3)
    Uq = fp4.quantize(r["U"].astype(np.float32), fmt, 0)
    Vq = fp4.quantize(r["V"].astype(np.float32), fmt, 0)
    low = (Uq.dequantize().T * r["S"]) @ Vq.dequantize()
    Rc = split.compensated_residual(A, Uq, r["S"], Vq)
    assert np.allclose(low + Rc, A, rtol=0, atol=1e-12)
    plain_err = np.linalg.norm(low + r["R"] - A)
    assert plain_err > 1e-3 * np.linalg.norm(A)
    e_plain = np.linalg.norm(low + fp4.quantize(r["R"].astype(np.float32), fmt, 1).dequantize() - A)
    e_comp = np.linalg.norm(low + fp4.quantize(Rc.astype(np.float32), fmt, 1).dequantize() - A)
    assert e_comp < e_plain
