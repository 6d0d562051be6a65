"""Pins for the oracle's re-quantized low-rank intermediates (reading R30):
the three-term expansion of a split x split product, the blocking axis of
each intermediate, exactness on representable intermediates, the own tensor
scale of each intermediate, zero padding of a short k, and the error bound of
the variant against the product with float32 intermediates."""
import numpy as np
import pytest

from oracle import fp4, gemm


def _q(x, fmt, axis):
    return fp4.quantize(np.asarray(x, dtype=np.float32), fmt, axis)


def _operands(fmt, M=64, N=96, K=128, ka=16, kb=32, seed=0):
    rng = np.random.default_rng(seed)
    A = rng.standard_normal((M, K))
    B = rng.standard_normal((K, N))
    PA, FA = rng.standard_normal((K, ka)) / np.sqrt(K), rng.standard_normal((M, ka)) / np.sqrt(M)
    PB, FB = rng.standard_normal((K, kb)) / np.sqrt(K), rng.standard_normal((N, kb)) / np.sqrt(N)
    opA = gemm.Operand(_q(A, fmt, 1), ka, _q(PA, fmt, 0), _q(FA, fmt, 0), np.linspace(6, 1, ka)) if ka else \
        gemm.Operand(_q(A, fmt, 1))
    opB = gemm.Operand(_q(B, fmt, 0), kb, _q(PB, fmt, 0), _q(FB, fmt, 0), np.linspace(5, 1, kb)) if kb else \
        gemm.Operand(_q(B, fmt, 0))
    return opA, opB


@pytest.mark.parametrize("ka,kb", [(16, 32), (0, 32), (16, 0), (8, 8)])
def test_intermediates_reassemble_the_product(ka, kb):
    opA, opB = _operands("nv", ka=ka, kb=kb)
    RA, RB, T1, FB, FA, T2 = gemm.intermediates(opA, opB)
    C = RA @ RB
    if T1 is not None:
        C = C + T1 @ FB.T
    if T2 is not None:
        C = C + FA @ T2
    # the dense product of the dequantized operands is formed another way
    want = gemm.gemm(opA, opB)
    assert np.max(np.abs(C - want)) <= 1e-12 * np.max(np.abs(want))
    assert (T1 is None) == (kb == 0) and (T2 is None) == (ka == 0)


def _block_bound(X, fmt, axis):
    """Per-entry bound of |deq(Q(X)) - X|: a quarter of the block maximum
    (E2M1's largest half step, 1 below 6 and saturation above, relative to a
    block maximum that maps to [4, 8) times the block scale); NVFP4 adds the
    E4M3 rounding of the block scale (at most 1/16 relative)."""
    bs = 32 if fmt == "mx" else 16
    Z = X if axis == 1 else X.T
    n = Z.shape[1]
    pad = (-n) % bs
    Zp = np.pad(np.abs(Z), ((0, 0), (0, pad)))
    bmax = Zp.reshape(Z.shape[0], -1, bs).max(axis=2)
    b = np.repeat(bmax, bs, axis=1)[:, :n] * (0.25 if fmt == "mx" else 0.25 * (1 + 1 / 16) + 1 / 16)
    return b if axis == 1 else b.T


@pytest.mark.parametrize("fmt", ["mx", "nv"])
def test_intermediates_are_blocked_along_their_contraction_axis(fmt):
    rng = np.random.default_rng(1)
    # magnitudes far apart: MXFP4's power-of-two block scales span any float32
    # range; NVFP4's E4M3 block scales span about 2^17 under one tensor scale,
    # so its rows stay within 2^12 of each other (every block scale normal)
    e = 20 if fmt == "mx" else 6
    # T1 (M x k_B): rows of different magnitude share no block when blocked along k_B
    T1 = (rng.standard_normal((64, 32)) * np.exp2(rng.integers(-e, e + 1, (64, 1)))).astype(np.float32)
    d = gemm.requantize(T1, fmt, 1)
    assert np.all(np.abs(d - T1) <= _block_bound(T1.astype(np.float64), fmt, 1))
    # T2 (k_A x N): columns of different magnitude, blocked along k_A
    T2 = (rng.standard_normal((32, 48)) * np.exp2(rng.integers(-e, e + 1, (1, 48)))).astype(np.float32)
    d2 = gemm.requantize(T2, fmt, 0)
    assert np.all(np.abs(d2 - T2) <= _block_bound(T2.astype(np.float64), fmt, 0))
    # the other axis would flush the small rows / columns to zero
    wrong = gemm.requantize(T1, fmt, 0)
    assert np.any(np.abs(wrong - T1) > _block_bound(T1.astype(np.float64), fmt, 1))


def test_representable_intermediates_pass_unchanged():
    # MXFP4 values (blocks along the contraction axis) re-quantize to themselves
    opA, opB = _operands("mx")
    RA, RB, T1, FB, FA, T2 = gemm.intermediates(opA, opB)
    X1 = gemm.requantize(np.float32(T1), "mx", 1).astype(np.float32)
    X2 = gemm.requantize(np.float32(T2), "mx", 0).astype(np.float32)
    assert np.array_equal(gemm.requantize(X1, "mx", 1), X1)
    assert np.array_equal(gemm.requantize(X2, "mx", 0), X2)
    got = gemm.gemm_requant(opA, opB, "mx", t1_32=X1, t2_32=X2)
    want = RA @ RB + X1.astype(np.float64) @ FB.T + FA @ X2.astype(np.float64)
    assert np.max(np.abs(got - want)) <= 1e-12 * np.max(np.abs(want))


def test_each_intermediate_has_its_own_tensor_scale():
    # NVFP4 quantization commutes with a power-of-two scale of the tensor:
    # the tensor scale follows the intermediate's own maximum
    rng = np.random.default_rng(2)
    T = rng.standard_normal((64, 32)).astype(np.float32)
    for e in (-30, 30):
        s = np.float32(2.0 ** e)
        assert np.array_equal(gemm.requantize(T * s, "nv", 1), gemm.requantize(T, "nv", 1) * np.float64(s))


@pytest.mark.parametrize("fmt", ["mx", "nv"])
def test_short_k_is_zero_padded(fmt):
    rng = np.random.default_rng(3)
    # small values: any non-zero padding would become the block maximum
    T = (rng.standard_normal((40, 8)) * 0.1).astype(np.float32)
    d = gemm.requantize(T, fmt, 1)
    assert d.shape == T.shape
    # the same values inside a full-width block of zeros quantize the same way
    bs = 32 if fmt == "mx" else 16
    full = np.zeros((40, bs), np.float32)
    full[:, :8] = T
    assert np.array_equal(d, fp4.quantize(full, fmt, 1).dequantize()[:, :8])
    d0 = gemm.requantize(T.T.copy(), fmt, 0)
    assert np.array_equal(d0, d.T)


@pytest.mark.parametrize("fmt", ["mx", "nv"])
def test_variant_error_within_the_block_bound(fmt):
    opA, opB = _operands(fmt, seed=4)
    RA, RB, T1, FB, FA, T2 = gemm.intermediates(opA, opB)
    base = RA @ RB + np.float32(T1).astype(np.float64) @ FB.T + FA @ np.float32(T2).astype(np.float64)
    var = gemm.gemm_requant(opA, opB, fmt)
    e1 = np.linalg.norm(_block_bound(np.float32(T1).astype(np.float64), fmt, 1))
    e2 = np.linalg.norm(_block_bound(np.float32(T2).astype(np.float64), fmt, 0))
    bound = e1 * np.linalg.norm(FB, 2) + np.linalg.norm(FA, 2) * e2
    err = np.linalg.norm(var - base)
    assert 0 < err <= bound
