"""GPU parity of the mean + spectral composite split (mean removal, then the
spectral split of the float32 mean-free residual, then the rank-(k + 1) FP4
factors) and of a forward product with the composite as the left operand.

The oracle is fed the GPU's own float32 mean (the mean itself is checked
against the float64 mean first), so every later comparison starts from the
same float32 residual: mean-free tap bit-exact, S, the rank-k part and R2
within 1e-3, FP4 factors and residual codes bit-exact on the GPU's own float32
values, the product within 2e-3 of the float64 product of the GPU's dequantized
operands."""
import numpy as np
import pytest
import torch

from oracle import averis, composite, fp4, gemm
from spectral_domain_quantization_b200 import api

from gpu_helpers import assert_fp4_equal, bf16_tensor, read_fp4, rel_fro

pytestmark = pytest.mark.gpu

TOL = 1e-3


def _data(m, n, r, seed):
    rng = np.random.default_rng(seed)
    mu = rng.standard_normal(n) * 4.0
    L = (rng.standard_normal((m, r)) * (8.0 / (1 + np.arange(r)))) @ rng.standard_normal((r, n)) / np.sqrt(n)
    return (mu[None, :] + L + 0.02 * rng.standard_normal((m, n))).astype(np.float32)


@pytest.mark.parametrize("fmt,dtype", [("nv", "bf16"), ("mx", "f32")])
def test_composite_split_and_forward(fmt, dtype):
    m, n, N, k, p = 512, 384, 256, 16, 8
    x = _data(m, n, 24, 7)
    if dtype == "bf16":
        X, xval = bf16_tensor(x)
    else:
        X, xval = torch.from_numpy(x).cuda(), x
    c = api.composite_split(X, k, p, 1, 3, fmt, rows=True, cols=True, tap=True)
    torch.cuda.synchronize()
    assert int(c.dev_status.cpu()[0]) == 0
    mu = c.mean.cpu().numpy()
    mu_ref = averis.column_mean(xval)
    assert np.max(np.abs(mu - mu_ref) / np.maximum(np.abs(mu_ref), 1e-3)) < 1e-6
    R1 = c.R1.cpu().numpy()
    assert np.array_equal(R1, averis.residual_f32(xval, mu))
    ref = composite.split(xval, k, p, 1, 3, mu32=mu)
    S = c.S.cpu().numpy().astype(np.float64)
    U = c.U.cpu().numpy().astype(np.float64)
    V = c.V.cpu().numpy().astype(np.float64)
    assert rel_fro(S, ref["S"]) < TOL
    assert rel_fro((U * S) @ V.T, (ref["U"] * ref["S"]) @ ref["V"].T) < TOL
    R2 = c.R2_f32.cpu().numpy()
    assert rel_fro(R2, ref["R2"]) < TOL
    # factors: [1 | U] and [mu | V] as quantized, bit-exact on the GPU's values
    F32 = c.F32.cpu().numpy()
    P32 = c.P32.cpu().numpy()
    assert np.array_equal(F32[:, 0], np.ones(m, np.float32)) and np.array_equal(P32[:, 0], mu)
    assert np.array_equal(F32[:, 1:], c.U.cpu().numpy()) and np.array_equal(P32[:, 1:], c.V.cpu().numpy())
    Fq, Pq = composite.factors_fp4(F32, P32, fmt)
    assert_fp4_equal(c.F_q, Fq, check_linear=False)
    assert_fp4_equal(c.P_q, Pq, check_linear=False)
    assert_fp4_equal(c.R_rows, fp4.quantize(R2, fmt, 1), check_linear=False)
    assert_fp4_equal(c.R_cols, fp4.quantize(R2, fmt, 0), check_linear=False)
    # Y = X W with X as the composite (rank k + 1 low-rank part)
    rng = np.random.default_rng(11)
    w32 = (rng.standard_normal((n, N)) * 0.05).astype(np.float32)
    qw = api.quantize_fp4(torch.from_numpy(np.ascontiguousarray(w32.T)).cuda(), fmt, 1)   # outer N, inner K
    y = api.linear_fwd(c.operand("left"), api.Operand(qw), m, N, n)
    torch.cuda.synchronize()
    left = gemm.Operand(read_fp4(c.R_rows), k + 1, read_fp4(c.P_q), read_fp4(c.F_q),
                        c.S1.cpu().numpy().astype(np.float64))
    want = gemm.gemm(left, gemm.Operand(read_fp4(qw)))
    assert rel_fro(y.cpu().numpy(), want) < 2e-3
    # and the composite is close to X itself (FP4 error only)
    assert rel_fro(gemm.dense_left(left), xval.astype(np.float64)) < 0.15   # FP4 error (MXFP4 ~0.11)
