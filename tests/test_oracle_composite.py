"""Pins for the oracle's mean + spectral composite split: reconstruction, exact
recovery of a mean plus a low-rank matrix, reduction to the plain spectral
split when the mean-free matrix is exact, the FP4 value of the ones column,
and the order of the two splits (mean first)."""
import numpy as np
import pytest

from oracle import averis, composite, fp4, split, gemm


def _rng(s):
    return np.random.default_rng(s)


def _mean_plus_lowrank(m, n, r, seed, noise=0.0):
    rng = _rng(seed)
    mu = rng.standard_normal(n) * 3.0
    L = (rng.standard_normal((m, r)) * (4.0 / (1 + np.arange(r)))) @ rng.standard_normal((r, n)) / np.sqrt(n)
    A = mu[None, :] + L + noise * rng.standard_normal((m, n))
    return A.astype(np.float32)


def test_reconstruction():
    A = _mean_plus_lowrank(160, 96, 12, 1, noise=0.05)
    parts = composite.split(A, 8, 8, 1, 5)
    # 1 mu^T + U S V^T + R2 equals the float32 input up to the float32
    # rounding of the mean-free residual
    err = np.linalg.norm(composite.reconstruct(parts) - A.astype(np.float64)) / np.linalg.norm(A)
    assert err < 1e-7
    # the low-rank part is rank k + 1 with the ones column and the mean first
    assert np.array_equal(parts["F"][:, 0], np.ones(160))
    assert np.array_equal(parts["P"][:, 0], parts["mu"].astype(np.float64))
    assert parts["S1"][0] == 1.0 and np.array_equal(parts["S1"][1:], parts["S"])


@pytest.mark.parametrize("q", [0, 1])
def test_mean_plus_exact_low_rank_recovered(q):
    # A = 1 mu^T + (rank 6): the spectral part of rank k = 8 takes all of the
    # mean-free matrix; R2 is float32 rounding only
    A = _mean_plus_lowrank(200, 120, 6, 2)
    parts = composite.split(A, 8, 8, q, 3)
    assert np.linalg.norm(parts["R2"]) / np.linalg.norm(parts["R1"]) < 1e-5


def test_zero_mean_reduces_to_spectral_split():
    # columns with exactly zero sums (rows in +/- pairs of dyadic values) and a
    # dyadic mean: fl32(a - mu) is exact, so the composite's U, S, V are the
    # plain split of the mean-free matrix with the same sketch
    rng = _rng(3)
    C = np.round(rng.standard_normal((64, 48)) * 64) / 64
    B = np.concatenate([C, -C], axis=0)
    mu = np.round(rng.standard_normal(48) * 8) / 8
    A = (B + mu[None, :]).astype(np.float32)
    assert np.array_equal(averis.column_mean(A), mu)
    parts = composite.split(A, 6, 6, 1, 9)
    assert np.array_equal(parts["R1"].astype(np.float64), B)
    ref = split.split(B, 6, 6, 1, 9)
    for key in ("U", "S", "V", "R"):
        got = parts["R2" if key == "R" else key]
        assert np.allclose(got, ref[key], rtol=0, atol=1e-12)


def test_mean_removed_before_the_spectral_split():
    # the same matrix split without removing the mean puts the mean into the
    # leading singular pair; the composite's leading pair is the mean-free one
    A = _mean_plus_lowrank(160, 96, 4, 4, noise=0.01)
    parts = composite.split(A, 4, 8, 1, 2)
    plain = split.split(A.astype(np.float64), 4, 8, 1, 2)
    mu = parts["mu"].astype(np.float64)
    cos_plain = abs(plain["V"][:, 0] @ mu) / np.linalg.norm(mu)
    cos_comp = abs(parts["V"][:, 0] @ mu) / np.linalg.norm(mu)
    assert cos_plain > 0.9 and cos_comp < 0.3


@pytest.mark.parametrize("fmt", ["nv", "mx"])
def test_ones_column_fp4_value(fmt):
    A = _mean_plus_lowrank(256, 128, 8, 5, noise=0.05)
    parts = composite.split(A, 8, 8, 1, 1)
    Fq, Pq = composite.factors_fp4(parts["F"].astype(np.float32), parts["P"].astype(np.float32), fmt)
    F = Fq.dequantize()
    if fmt == "mx":
        assert np.array_equal(F[0], np.ones(256))
    else:
        # 6 (E2M1) x 448 (E4M3) x fl32(1 / 2688): U's entries are below 1, so
        # the ones set the tensor maximum
        one = 2688.0 * np.float64(np.float32(1.0) / np.float32(2688.0))
        assert np.array_equal(F[0], np.full(256, one))
        assert abs(one - 1.0) <= 2.0 ** -24
    # the composite as a left operand of a product: the dense value is
    # 1 mu~^T + U~ S V~^T + R2~ with the quantized pieces
    R2q = fp4.quantize(parts["R2"].astype(np.float32), fmt, 1)
    op = gemm.Operand(R2q, 9, Pq, Fq, parts["S1"])
    dense = gemm.dense_left(op)
    assert np.linalg.norm(dense - A) / np.linalg.norm(A) < 0.15
