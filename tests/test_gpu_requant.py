"""GPU parity of the FP4 re-quantized low-rank intermediates (reading R30):
the product with T1 (and T2) re-quantized to FP4 along k against the oracle's
gemm_requant, within 2e-3; and its accuracy cost against the product with
float32 intermediates (the relative errors against the oracle's product of
the same FP4 operands with exact intermediates are printed).

Both sides quantize float32 intermediates: the device's T1 = R_A P_B + ...
(accumulated in float32 on the tensor cores) and the oracle's fl32 of the
exact T1.  The two can differ in the last bits, so a value that lies within
that distance of an FP4 rounding boundary may take the neighbouring code on
one side; such flips are rare and move the product by far less than the
tolerance."""
import numpy as np
import pytest
import torch

from oracle import fp4, gemm
from spectral_domain_quantization_b200 import api

from gpu_helpers import assert_fp4_equal, rel_fro

pytestmark = pytest.mark.gpu

TOL = 2e-3


def _rand(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape) * scale
    x *= np.exp2(rng.integers(-2, 3, (shape[0], 1)))
    return x.astype(np.float32)


def _q(x, fmt, axis):
    q = api.quantize_fp4(torch.from_numpy(x).cuda(), fmt, axis)
    ref = fp4.quantize(x, fmt, axis)
    torch.cuda.synchronize()
    assert_fp4_equal(q, ref, check_linear=False)
    return q, ref


def _factors(n_free, K, k, fmt, seed):
    P = (_rand((K, k), seed) / np.sqrt(K)).astype(np.float32)
    F = (_rand((n_free, k), seed + 1) / np.sqrt(n_free)).astype(np.float32)
    S = np.linspace(8, 1, k).astype(np.float32)
    qP, rP = _q(P, fmt, 0)
    qF, rF = _q(F, fmt, 0)
    return qP, rP, qF, rF, S


@pytest.mark.parametrize("fmt", ["mx", "nv"])
@pytest.mark.parametrize("M,N,K,kb", [(256, 512, 512, 8), (300, 288, 1024, 64), (2000, 2560, 512, 64)])
def test_requant_right_split_product(fmt, M, N, K, kb):
    qa, ra = _q(_rand((M, K), 7), fmt, 1)
    qr, rr = _q(_rand((K, N), 8, 0.1), fmt, 0)
    qP, rP, qF, rF, S = _factors(N, K, kb, fmt, 9)
    St = torch.from_numpy(S).cuda()
    y = api.linear_fwd(api.Operand(qa), api.Operand(qr, kb, qP, qF, St, requant=True), M, N, K)
    y0 = api.linear_fwd(api.Operand(qa), api.Operand(qr, kb, qP, qF, St), M, N, K)
    torch.cuda.synchronize()
    opA, opB = gemm.Operand(ra), gemm.Operand(rr, kb, rP, rF, S)
    want = gemm.gemm_requant(opA, opB, fmt)
    assert rel_fro(y.cpu().numpy(), want) < TOL
    # accuracy cost: the variant moves the product, the base path does not
    exact = gemm.gemm(opA, opB)
    e0, e1 = rel_fro(y0.cpu().numpy(), exact), rel_fro(y.cpu().numpy(), exact)
    print(f"requant cost {fmt} M={M} N={N} K={K} k={kb}: float32 intermediates {e0:.2e}, FP4 {e1:.2e}")
    assert e0 < TOL
    assert e1 > e0


@pytest.mark.parametrize("fmt", ["mx", "nv"])
def test_requant_both_split_product(fmt):
    M, N, K, ka, kb = 384, 512, 1024, 16, 64
    qra, rra = _q(_rand((M, K), 11, 0.2), fmt, 1)
    qPa, rPa, qFa, rFa, Sa = _factors(M, K, ka, fmt, 12)
    qrb, rrb = _q(_rand((K, N), 13, 0.2), fmt, 0)
    qPb, rPb, qFb, rFb, Sb = _factors(N, K, kb, fmt, 14)
    y = api.linear_fwd(api.Operand(qra, ka, qPa, qFa, torch.from_numpy(Sa).cuda(), requant=True),
                       api.Operand(qrb, kb, qPb, qFb, torch.from_numpy(Sb).cuda(), requant=True), M, N, K)
    torch.cuda.synchronize()
    want = gemm.gemm_requant(gemm.Operand(rra, ka, rPa, rFa, Sa), gemm.Operand(rrb, kb, rPb, rFb, Sb), fmt)
    assert rel_fro(y.cpu().numpy(), want) < TOL
