"""GPU parity of the FP4 products (metis_linear_fwd / metis_linear_bwd)
against the oracle's float64 product of the dequantized operands.

The operands are quantized independently on both sides from the same seeded
float32 data; the test first asserts the two quantizations are bit-identical,
so both products see the same operands.  Contract: relative Frobenius error
<= 2e-3; the plain FP4 product is held to 1e-5 (fp32 accumulation only)."""
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


def _q(x, fmt, axis, inner_sum=False):
    """Quantize on both sides, assert equality, return (gpu QTensor, oracle FP4Tensor)."""
    t = torch.from_numpy(x).cuda()
    q = api.quantize_fp4(t, fmt, axis, inner_sum=inner_sum)
    ref = fp4.quantize(x, fmt, axis)
    torch.cuda.synchronize()
    assert_fp4_equal(q, ref, check_linear=False)
    return q, ref


@pytest.mark.parametrize("fmt", ["mx", "nv"])
@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (300, 520, 1056), (1000, 64, 512),
                                   (200, 100, 320), (129, 384, 4096)])
def test_plain_product(fmt, M, N, K):
    a = _rand((M, K), M + K)
    b = _rand((K, N), N + K + 1)
    qa, ra = _q(a, fmt, 1)
    qb, rb = _q(b, fmt, 0)
    y = api.linear_fwd(api.Operand(qa), api.Operand(qb), M, N, K)
    torch.cuda.synchronize()
    want = gemm.gemm(gemm.Operand(ra), gemm.Operand(rb))
    err = rel_fro(y.cpu().numpy(), want)
    assert err < 1e-5, err


@pytest.mark.parametrize("M,N,K", [(256, 512, 1024), (128, 512, 1024), (300, 200, 512)])
def test_plain_product_bf16_output(M, N, K):
    # the bf16 output is the float32 output of the same call rounded once,
    # and the float32 output meets the product tolerance
    qa, ra = _q(_rand((M, K), 1), "nv", 1)
    qb, rb = _q(_rand((K, N), 2), "nv", 0)
    y16 = api.linear_fwd(api.Operand(qa), api.Operand(qb), M, N, K, out_dtype=torch.bfloat16)
    y = api.linear_fwd(api.Operand(qa), api.Operand(qb), M, N, K)
    torch.cuda.synchronize()
    want = gemm.gemm(gemm.Operand(ra), gemm.Operand(rb))
    assert rel_fro(y.cpu().numpy(), want) < 1e-5
    assert torch.equal(y16.cpu(), y.cpu().to(torch.bfloat16))


# Shapes whose rounds of tiles over 148 SMs favour the 256 x 192 tile (two
# 128-row halves sharing one B tile): full-width and ragged tiles, rows of C
# with and without 16-byte alignment.
WIDE_SHAPES = [(2048, 2560, 512), (2000, 2500, 512)]


@pytest.mark.parametrize("fmt", ["mx", "nv"])
@pytest.mark.parametrize("M,N,K", WIDE_SHAPES)
def test_wide_tile_product(fmt, M, N, K):
    a = _rand((M, K), M + 3)
    b = _rand((K, N), N + 5)
    qa, ra = _q(a, fmt, 1)
    qb, rb = _q(b, fmt, 0)
    y = api.linear_fwd(api.Operand(qa), api.Operand(qb), M, N, K)
    y16 = api.linear_fwd(api.Operand(qa), api.Operand(qb), M, N, K, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    want = gemm.gemm(gemm.Operand(ra), gemm.Operand(rb))
    assert rel_fro(y.cpu().numpy(), want) < 1e-5
    # the bf16 output is the float32 one rounded once (same accumulation)
    assert torch.equal(y16.cpu(), y.cpu().to(torch.bfloat16))


@pytest.mark.parametrize("fmt", ["mx", "nv"])
def test_wide_tile_right_split_product(fmt):
    # the low-rank chunks appended to the K loop of the wide tile
    M, N, K, kb = 2000, 2560, 512, 64
    qa, ra = _q(_rand((M, K), 17), fmt, 1)
    qr, rr = _q(_rand((K, N), 18, 0.1), fmt, 0)
    qP, rP, qF, rF, S = _factors(N, K, kb, fmt, 19)
    y = api.linear_fwd(api.Operand(qa), api.Operand(qr, kb, qP, qF, torch.from_numpy(S).cuda()), M, N, K)
    torch.cuda.synchronize()
    want = gemm.gemm(gemm.Operand(ra), gemm.Operand(rr, kb, rP, rF, S))
    assert rel_fro(y.cpu().numpy(), want) < TOL


def _factors(n_free, K, k, fmt, seed):
    P = (_rand((K, k), seed) / np.sqrt(K)).astype(np.float32)
    F = (_rand((n_free, k), seed + 1) / np.sqrt(n_free)).astype(np.float32)
    S = (np.linspace(8, 1, k)).astype(np.float32)
    qP, rP = _q(P, fmt, 0)
    qF, rF = _q(F, fmt, 0)
    return qP, rP, qF, rF, S


@pytest.mark.parametrize("fmt", ["mx", "nv"])
@pytest.mark.parametrize("M,N,K,kb", [(256, 512, 512, 8), (300, 288, 1024, 64), (128, 1024, 4096, 64)])
def test_right_split_product(fmt, M, N, K, kb):
    # forward of a split weight: Y = X_q (R_q + P S F^T)
    qa, ra = _q(_rand((M, K), 7), fmt, 1)
    qr, rr = _q(_rand((K, N), 8, 0.1), fmt, 0)
    qP, rP, qF, rF, S = _factors(N, K, kb, fmt, 9)
    St = torch.from_numpy(S).cuda()
    y = api.linear_fwd(api.Operand(qa), api.Operand(qr, kb, qP, qF, St), M, N, K)
    torch.cuda.synchronize()
    want = gemm.gemm(gemm.Operand(ra), gemm.Operand(rr, kb, rP, rF, S))
    assert rel_fro(y.cpu().numpy(), want) < TOL


@pytest.mark.parametrize("fmt", ["mx", "nv"])
def test_both_split_product(fmt):
    M, N, K, ka, kb = 384, 512, 1024, 16, 64
    qra, rra = _q(_rand((M, K), 11, 0.2), fmt, 1)
    qPa, rPa, qFa, rFa, Sa = _factors(M, K, ka, fmt, 12)
    qrb, rrb = _q(_rand((K, N), 13, 0.2), fmt, 0)
    qPb, rPb, qFb, rFb, Sb = _factors(N, K, kb, fmt, 14)
    y = api.linear_fwd(api.Operand(qra, ka, qPa, qFa, torch.from_numpy(Sa).cuda()),
                       api.Operand(qrb, kb, qPb, qFb, torch.from_numpy(Sb).cuda()), M, N, K)
    torch.cuda.synchronize()
    want = gemm.gemm(gemm.Operand(rra, ka, rPa, rFa, Sa), gemm.Operand(rrb, kb, rPb, rFb, Sb))
    assert rel_fro(y.cpu().numpy(), want) < TOL


@pytest.mark.parametrize("fmt,K", [("nv", 1536), ("mx", 20480)])
def test_both_split_core_product(fmt, K):
    # P_A and P_B share their first 13 columns, so C_ab = P_A^T P_B is O(1)
    # and the F_A S_A C_ab S_B F_B^T term carries most of C; an odd
    # ka = 13 next to the largest kb = 128, and at K = 20480 each partial of
    # C_ab covers two rounds of 64 positions
    M, N, ka, kb = 256, 384, 13, 128
    P = (_rand((K, kb), 61) / np.sqrt(K)).astype(np.float32)
    Fa = (_rand((M, 16), 62) / np.sqrt(M)).astype(np.float32)
    # the 13 leading columns are quantized as strided views (row stride 16
    # and 128 floats keeps 16-byte rows)
    qPa = api.quantize_fp4(torch.from_numpy(P).cuda()[:, :ka], fmt, 0)
    qFa = api.quantize_fp4(torch.from_numpy(Fa).cuda()[:, :ka], fmt, 0)
    rPa, rFa = fp4.quantize(P[:, :ka], fmt, 0), fp4.quantize(Fa[:, :ka], fmt, 0)
    torch.cuda.synchronize()
    assert_fp4_equal(qPa, rPa, check_linear=False)
    assert_fp4_equal(qFa, rFa, check_linear=False)
    qPb, rPb = _q(P, fmt, 0)
    qFb, rFb = _q((_rand((N, kb), 63) / np.sqrt(N)).astype(np.float32), fmt, 0)
    Sa = np.linspace(8, 1, ka).astype(np.float32)
    Sb = np.linspace(6, 1, kb).astype(np.float32)
    qra, rra = _q(_rand((M, K), 64, 0.02), fmt, 1)
    qrb, rrb = _q(_rand((K, N), 65, 0.02), fmt, 0)
    y = api.linear_fwd(api.Operand(qra, ka, qPa, qFa, torch.from_numpy(Sa).cuda()),
                       api.Operand(qrb, kb, qPb, qFb, torch.from_numpy(Sb).cuda()), M, N, K)
    torch.cuda.synchronize()
    A = gemm.Operand(rra, ka, rPa, rFa, Sa)
    B = gemm.Operand(rrb, kb, rPb, rFb, Sb)
    want = gemm.gemm(A, B)
    # the core term is most of the product
    core = gemm.gemm(gemm.Operand(rra), gemm.Operand(rrb))
    assert np.linalg.norm(want - core) > 2 * np.linalg.norm(core)
    assert rel_fro(y.cpu().numpy(), want) < TOL


def test_both_split_many_tiles_per_cta():
    # both operands split at rank 64: four low-rank chunks, as many as the
    # 128x256 kernel's ring has stages, and about two tiles per CTA, so the
    # scale copies of a tile's first K step follow a full round of low-rank
    # stages; the low-rank part carries most of C
    fmt = "nv"
    M, N, K, k = 4096, 2048, 1024, 64
    P = (_rand((K, k), 71) / np.sqrt(K)).astype(np.float32)
    qPa, rPa = _q(P, fmt, 0)
    qPb, rPb = qPa, rPa
    qFa, rFa = _q((_rand((M, k), 72) / np.sqrt(M)).astype(np.float32), fmt, 0)
    qFb, rFb = _q((_rand((N, k), 73) / np.sqrt(N)).astype(np.float32), fmt, 0)
    Sa = np.linspace(8, 1, k).astype(np.float32)
    Sb = np.linspace(6, 1, k).astype(np.float32)
    qra, rra = _q(_rand((M, K), 74, 0.05), fmt, 1)
    qrb, rrb = _q(_rand((K, N), 75, 0.05), fmt, 0)
    y = api.linear_fwd(api.Operand(qra, k, qPa, qFa, torch.from_numpy(Sa).cuda()),
                       api.Operand(qrb, k, qPb, qFb, torch.from_numpy(Sb).cuda()), M, N, K)
    torch.cuda.synchronize()
    want = gemm.gemm(gemm.Operand(rra, k, rPa, rFa, Sa), gemm.Operand(rrb, k, rPb, rFb, Sb))
    assert rel_fro(y.cpu().numpy(), want) < TOL


def test_both_split_long_contraction():
    # K = 14336 (56 K tiles) with few output tiles: the low-rank products run
    # split-K with a split count that does not divide the K tiles evenly
    fmt = "nv"
    M, N, K, ka, kb = 128, 4096, 14336, 64, 64
    qra, rra = _q(_rand((M, K), 51, 0.2), fmt, 1)
    qPa, rPa, qFa, rFa, Sa = _factors(M, K, ka, fmt, 52)
    qrb, rrb = _q(_rand((K, N), 53, 0.02), fmt, 0)
    qPb, rPb, qFb, rFb, Sb = _factors(N, K, kb, fmt, 54)
    y = api.linear_fwd(api.Operand(qra, ka, qPa, qFa, torch.from_numpy(Sa).cuda()),
                       api.Operand(qrb, kb, qPb, qFb, torch.from_numpy(Sb).cuda()), M, N, K)
    torch.cuda.synchronize()
    want = gemm.gemm(gemm.Operand(rra, ka, rPa, rFa, Sa), gemm.Operand(rrb, kb, rPb, rFb, Sb))
    assert rel_fro(y.cpu().numpy(), want) < TOL


def test_averis_ones_factors():
    # left operand X = 1 mu^T + R (F = ones), right operand plain; and the dW
    # form X^T dY with both means (P = ones on both sides)
    fmt = "nv"
    M, N, K = 512, 256, 768
    x = _rand((M, K), 21)
    mu = (np.random.default_rng(22).standard_normal(K) * 5).astype(np.float32)
    qr, rr = _q(x, fmt, 1)
    qmu, rmu = _q(mu[None, :].copy(), fmt, 1)          # outer 1, inner K
    qw, rw = _q(_rand((K, N), 23, 0.02), fmt, 0, inner_sum=True)
    y = api.linear_fwd(api.Operand(qr, 1, qmu, None, None), api.Operand(qw), M, N, K)
    torch.cuda.synchronize()
    want = gemm.gemm(gemm.Operand(rr, 1, rmu, "ones", [1.0]), gemm.Operand(rw))
    assert rel_fro(y.cpu().numpy(), want) < TOL
    # dW = X^T dY: A = X^T (K x M), contraction M; X^T = mu 1^T + R^T: P = ones, F = mu
    dy = _rand((M, N), 24, 0.01)
    nu = (np.random.default_rng(25).standard_normal(N) * 0.01).astype(np.float32)
    qxt, rxt = _q(x, fmt, 0, inner_sum=True)            # outer K, inner M
    qdy, rdy = _q(dy, fmt, 0, inner_sum=True)           # outer N, inner M
    qnu, rnu = _q(nu[None, :].copy(), fmt, 1)           # outer 1, inner N
    dw = api.linear_fwd(api.Operand(qxt, 1, None, qmu, None), api.Operand(qdy, 1, None, qnu, None), K, N, M)
    torch.cuda.synchronize()
    want = gemm.gemm(gemm.Operand(rxt, 1, "ones", rmu, [1.0]), gemm.Operand(rdy, 1, "ones", rnu, [1.0]))
    assert rel_fro(dw.cpu().numpy(), want) < TOL


def test_backward_products():
    fmt = "mx"
    M, N, K, k = 256, 384, 512, 16
    w = _rand((K, N), 31, 0.05)
    dy = _rand((M, N), 32, 0.01)
    x = _rand((M, K), 33)
    # dX = dY W^T: left dY quantized along N, right W^T with residual along N
    qdy_n, rdy_n = _q(dy, fmt, 1)
    qw_n, rw_n = _q(w, fmt, 1)                          # outer K, inner N
    U = (_rand((K, k), 34) / np.sqrt(K)).astype(np.float32)
    V = (_rand((N, k), 35) / np.sqrt(N)).astype(np.float32)
    S = np.linspace(4, 1, k).astype(np.float32)
    qU, rU = _q(U, fmt, 0)                              # outer k, inner K
    qV, rV = _q(V, fmt, 0)                              # outer k, inner N
    # dW = X^T dY: left X^T (quantized along M), right dY along M
    qx_m, rx_m = _q(x, fmt, 0)
    qdy_m, rdy_m = _q(dy, fmt, 0)
    St = torch.from_numpy(S).cuda()
    dX, dW = api.linear_bwd(api.Operand(qdy_n), api.Operand(qw_n, k, qV, qU, St),
                            api.Operand(qx_m), api.Operand(qdy_m), M, N, K)
    torch.cuda.synchronize()
    want_dx = gemm.gemm(gemm.Operand(rdy_n), gemm.Operand(rw_n, k, rV, rU, S))
    want_dw = gemm.gemm(gemm.Operand(rx_m), gemm.Operand(rdy_m))
    assert rel_fro(dX.cpu().numpy(), want_dx) < TOL
    assert rel_fro(dW.cpu().numpy(), want_dw) < 1e-5


def test_full_size_forward_sampled_rows():
    # the single-layer workload's product shape 8192 x 4096 x 4096 (NVFP4),
    # checked on 256 sampled output rows
    M, N, K = 8192, 4096, 4096
    rng = np.random.default_rng(41)
    a = rng.standard_normal((M, K), dtype=np.float32)
    b = (rng.standard_normal((K, N), dtype=np.float32) * 0.02).astype(np.float32)
    qa, ra = _q(a, "nv", 1)
    qb, rb = _q(b, "nv", 0)
    y = api.linear_fwd(api.Operand(qa), api.Operand(qb), M, N, K)
    torch.cuda.synchronize()
    rows = np.sort(rng.choice(M, 256, replace=False))
    want = gemm.gemm(gemm.Operand(ra), gemm.Operand(rb), rows=rows)
    assert rel_fro(y.cpu().numpy()[rows], want) < 1e-5
