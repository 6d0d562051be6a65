"""GPU parity of averis_split and of the Averis forward / backward products.

mean within float32 rounding of the oracle's float64 mean; residual FP4
(both axes) and mean FP4 bit-exact against the oracle quantizer fed the
GPU's float32 mean; residual inner sums within float32 summation error; the
W4A4G4 products with Averis operands within 2e-3 of the oracle's float64
product of the dequantized operands."""
import numpy as np
import pytest
import torch

from oracle import averis, fp4, gemm
from spectral_domain_quantization_b200 import api, inputs

from gpu_helpers import assert_fp4_equal, rel_fro, to_device

pytestmark = pytest.mark.gpu


def _check_split(X32, res, fmt):
    mu = res.mean.cpu().numpy()
    mu_ref, _ = averis.split(X32.astype(np.float64))
    assert np.max(np.abs(mu - mu_ref) / np.maximum(np.abs(mu_ref), 1e-3)) < 1e-6
    r32 = averis.residual_f32(X32, mu)
    ref_rows = fp4.quantize(r32, fmt, 1)
    ref_cols = fp4.quantize(r32, fmt, 0)
    if fmt == "nv":
        # the residual's tensor maximum comes from the column extremes
        assert averis.residual_amax_from_columns(X32, mu) == np.abs(r32).max()
    assert_fp4_equal(res.R_rows, ref_rows, check_linear=False)
    assert_fp4_equal(res.R_cols, ref_cols, check_linear=False)
    assert_fp4_equal(res.mean_q, fp4.quantize(mu[None, :].copy(), fmt, 1), check_linear=False)
    assert rel_fro(res.R_cols.inner_sum.cpu().numpy(), ref_cols.colsum()) < 1e-5
    if res.R_f32 is not None:
        assert np.array_equal(res.R_f32.cpu().numpy(), r32)
    return ref_rows, ref_cols


@pytest.mark.parametrize("fmt", ["nv", "mx"])
@pytest.mark.parametrize("shape", [(4096, 256), (352, 160), (32, 96)])
def test_averis_split_parity(fmt, shape):
    m, n = shape
    d = inputs.make("averis_32768", scale=dict(M=m, K=n, N=64))
    X = to_device(d["X"])
    res = api.averis_split(X, fmt, tap=True)
    torch.cuda.synchronize()
    _check_split(d["X"].f32(), res, fmt)


def test_averis_pure_mean_input():
    mu0 = np.linspace(-3, 5, 64).astype(np.float32)
    X = np.tile(mu0, (1024, 1))
    res = api.averis_split(torch.from_numpy(X).cuda(), "nv", tap=True)
    torch.cuda.synchronize()
    assert np.array_equal(res.mean.cpu().numpy(), mu0)
    assert np.all(res.R_f32.cpu().numpy() == 0)
    assert np.all(res.R_rows.codes.cpu().numpy() == 0)


def test_averis_layer_forward_backward():
    # the Averis workload at 2048 x 512 (N = 384): Y = X W, dX = dY W^T,
    # dW = X^T dY with X and dY split into mean + residual, W plain NVFP4
    M, K, N = 2048, 512, 384
    d = inputs.make("averis_32768", scale=dict(M=M, K=K, N=N))
    X, W, dY = to_device(d["X"]), to_device(d["W"]), to_device(d["dY"])
    ax = api.averis_split(X, "nv")
    ady = api.averis_split(dY, "nv")
    wk = api.quantize_fp4(W, "nv", 0)                # outer N, inner K (forward)
    wn = api.quantize_fp4(W, "nv", 1, inner_sum=True)  # outer K, inner N (dX)
    Y = api.linear_fwd(ax.left(), api.Operand(wk), M, N, K)
    dX, dW = api.linear_bwd(ady.left(), api.Operand(wn), ax.left_t(), ady.right_m(), M, N, K)
    torch.cuda.synchronize()
    x32, dy32 = d["X"].f32(), d["dY"].f32()
    mx = ax.mean.cpu().numpy()
    my = ady.mean.cpu().numpy()
    rx_r, rx_c = fp4.quantize(averis.residual_f32(x32, mx), "nv", 1), fp4.quantize(averis.residual_f32(x32, mx), "nv", 0)
    ry_r, ry_c = fp4.quantize(averis.residual_f32(dy32, my), "nv", 1), fp4.quantize(averis.residual_f32(dy32, my), "nv", 0)
    qmx, qmy = fp4.quantize(mx[None, :].copy(), "nv", 1), fp4.quantize(my[None, :].copy(), "nv", 1)
    w32 = d["W"].f32()
    rwk, rwn = fp4.quantize(w32, "nv", 0), fp4.quantize(w32, "nv", 1)
    want_y = gemm.gemm(gemm.Operand(rx_r, 1, qmx, "ones", [1.0]), gemm.Operand(rwk))
    want_dx = gemm.gemm(gemm.Operand(ry_r, 1, qmy, "ones", [1.0]), gemm.Operand(rwn))
    want_dw = gemm.gemm(gemm.Operand(rx_c, 1, "ones", qmx, [1.0]), gemm.Operand(ry_c, 1, "ones", qmy, [1.0]))
    assert rel_fro(Y.cpu().numpy(), want_y) < 2e-3
    assert rel_fro(dX.cpu().numpy(), want_dx) < 2e-3
    assert rel_fro(dW.cpu().numpy(), want_dw) < 2e-3
