"""GPU parity of metis_split against the oracle's randomized split.

Checks (reading R8): singular values S, the rank-k part L = U S V^T and the
residual R within relative Frobenius 1e-3; U, V column by column where the
singular values are well separated; FP4 outputs (U_q, V_q, R along both axes)
bit-exact against the oracle quantizer fed the GPU's own float32 U, V and R."""
import numpy as np
import pytest
import torch

from oracle import fp4, sketch, split
from spectral_domain_quantization_b200 import api, inputs

from gpu_helpers import assert_fp4_equal, read_fp4, rel_fro, to_device

pytestmark = pytest.mark.gpu

TOL = 1e-3


def _check(A64, res, ref, fmt, check_vectors=True, r_tol=TOL, tap_scale=None):
    U = res.U.cpu().numpy().astype(np.float64)
    S = res.S.cpu().numpy().astype(np.float64)
    V = res.V.cpu().numpy().astype(np.float64)
    assert int(res.dev_status.cpu()[0]) == 0
    assert rel_fro(S, ref["S"]) < TOL
    L = (U * S) @ V.T
    Lref = (ref["U"] * ref["S"]) @ ref["V"].T
    assert rel_fro(L, Lref) < TOL
    R = res.R_f32.cpu().numpy()
    assert rel_fro(R, ref["R"]) < r_tol
    # the tap is A - U S V^T, with U S V^T from bf16 hi/lo products (about
    # 2^-16 of |L|): relative to |R|, or to tap_scale where |R| << |L|
    den = np.linalg.norm(R) if tap_scale is None else tap_scale
    assert np.linalg.norm(R.astype(np.float64) - (A64 - L)) / den < 1e-5
    if check_vectors:
        # a singular vector is unique (up to the sign both sides fix the same
        # way) only where its value is separated from its neighbours; there
        # the columns are held to the factor tolerance
        s = ref["S"]
        gap = np.minimum(np.abs(np.diff(np.r_[np.inf, s])), np.abs(np.diff(np.r_[s, -np.inf])))
        sep = gap / s > 0.05
        for j in np.flatnonzero(sep):
            assert rel_fro(U[:, j], ref["U"][:, j]) < TOL, j
            assert rel_fro(V[:, j], ref["V"][:, j]) < TOL, j
    # FP4 outputs: bit-exact on the GPU's own float32 values
    k = U.shape[1]
    assert_fp4_equal(res.U_q, fp4.quantize(res.U.cpu().numpy(), fmt, 0), check_linear=False)
    assert_fp4_equal(res.V_q, fp4.quantize(res.V.cpu().numpy(), fmt, 0), check_linear=False)
    assert_fp4_equal(res.R_rows, fp4.quantize(R, fmt, 1), check_linear=False)
    assert_fp4_equal(res.R_cols, fp4.quantize(R, fmt, 0), check_linear=False)


def test_split_tiny_workload():
    d = inputs.make("tiny_256")
    c = d["cfg"]
    A = to_device(d["W"])
    res = api.split(A, c["k"], c["p"], c["q"], c["sketch_seed"], c["fmt"], tap=True)
    torch.cuda.synchronize()
    A64 = d["W"].f64()
    ref = split.split(A64, c["k"], c["p"], c["q"], c["sketch_seed"])
    _check(A64, res, ref, c["fmt"])


def test_split_exact_rank_recovered():
    rng = np.random.default_rng(3)
    A = (rng.standard_normal((192, 6)) @ rng.standard_normal((6, 160))).astype(np.float32)
    res = api.split(torch.from_numpy(A).cuda(), 8, 8, 1, 7, "mx", tap=True)
    torch.cuda.synchronize()
    R = res.R_f32.cpu().numpy()
    assert np.linalg.norm(R) / np.linalg.norm(A) < 1e-5
    ref = split.split(A.astype(np.float64), 8, 8, 1, 7)
    L = (res.U.cpu().numpy().astype(np.float64) * res.S.cpu().numpy()) @ res.V.cpu().numpy().T
    assert rel_fro(L, (ref["U"] * ref["S"]) @ ref["V"].T) < TOL


@pytest.mark.parametrize("fmt", ["nv", "mx"])
def test_split_layer_shape_reduced(fmt):
    # the single-layer recipe at 512 x 768 (several tiles), k=64, p=16, q=1
    d = inputs.make("layer_4096", scale=dict(K=512, N=768, M=128))
    A = to_device(d["W"])
    res = api.split(A, 64, 16, 1, 0, fmt, tap=True)
    torch.cuda.synchronize()
    A64 = d["W"].f64()
    ref = split.split(A64, 64, 16, 1, 0)
    _check(A64, res, ref, fmt)


@pytest.mark.parametrize("q", [0, 2])
def test_split_power_iterations(q):
    d = inputs.make("layer_4096", scale=dict(K=384, N=256, M=128))
    A = to_device(d["W"])
    res = api.split(A, 16, 16, q, 5, "nv", tap=True)
    torch.cuda.synchronize()
    A64 = d["W"].f64()
    _check(A64, res, split.split(A64, 16, 16, q, 5), "nv")


@pytest.mark.parametrize("q", [0, 1])
def test_split_eight_slice_sketch(q):
    # W 2048 x 4096: the sketch pass runs 8 K slices per 128-row tile (each
    # CTA of the cluster finishes 16 rows); the 4096-row passes run 4 slices
    d = inputs.make("layer_4096", scale=dict(K=2048, N=4096, M=128))
    A = to_device(d["W"])
    res = api.split(A, 16, 16, q, 2, "nv", tap=True)
    torch.cuda.synchronize()
    A64 = d["W"].f64()
    _check(A64, res, split.split(A64, 16, 16, q, 2), "nv")


def test_split_sampled_sparse_sign():
    # the sampled-activation recipe at 4096 x 512: 256 rows, sparse sign (4), k=32, p=16
    d = inputs.make("sampled_65536", scale=dict(M=4096, K=512))
    A = to_device(d["A"])
    res = api.split(A, 32, 16, 0, 0, "mx", sketch="sparse_sign", nnz=4, sample_rows=256, tap=True)
    torch.cuda.synchronize()
    assert np.array_equal(res.idx.cpu().numpy(), sketch.sample_rows(4096, 256, 0))
    A64 = d["A"].f64()
    ref = split.split(A64, 32, 16, 0, 0, kind="sparse_sign", nnz=4, sample_rows=256)
    _check(A64, res, ref, "mx", check_vectors=False)


def test_split_full_size_layer_weight():
    # W 4096 x 4096 of the single-layer workload, NVFP4, k=64, p=16, q=1
    d = inputs.make("layer_4096")
    c = d["cfg"]
    A = to_device(d["W"])
    res = api.split(A, c["k"], c["p"], c["q"], c["sketch_seed"], "nv", tap=True)
    torch.cuda.synchronize()
    A64 = d["W"].f64()
    ref = split.split(A64, c["k"], c["p"], c["q"], c["sketch_seed"])
    _check(A64, res, ref, "nv")


@pytest.mark.parametrize("k,p", [(96, 16), (92, 3)])
def test_split_largest_cores(k, p):
    # the largest core (l = 112) and an odd l = 95 (padded to 96): a
    # 384 x 256 matrix with geometric singular values 2^(-i/16) (4 % gaps),
    # so the rank-k part is well determined at k = 92 and 96
    rng = np.random.default_rng(11)
    Ul, _ = np.linalg.qr(rng.standard_normal((384, 256)))
    Vr, _ = np.linalg.qr(rng.standard_normal((256, 256)))
    A64 = (Ul * 2.0 ** (-np.arange(256) / 16.0)) @ Vr.T
    A = A64.astype(np.float32)
    res = api.split(torch.from_numpy(A).cuda(), k, p, 1, 3, "nv", tap=True)
    torch.cuda.synchronize()
    A64 = A.astype(np.float64)
    _check(A64, res, split.split(A64, k, p, 1, 3), "nv", tap_scale=np.linalg.norm(A64))


@pytest.mark.parametrize("fmt", ["nv", "mx"])
def test_split_compensated_residual(fmt):
    # R = A - deq(U_q) S deq(V_q)^T against the oracle fed the GPU's own FP4
    # factors; U, S, V and their codes are those of the plain split; the
    # quantized operand R_q + deq(U_q) S deq(V_q)^T is closer to A than with
    # the plain residual
    d = inputs.make("layer_4096", scale=dict(K=512, N=768, M=128))
    A = to_device(d["W"])
    plain = api.split(A, 64, 16, 1, 0, fmt, tap=True)
    comp = api.split(A, 64, 16, 1, 0, fmt, tap=True, compensate=True)
    torch.cuda.synchronize()
    assert int(comp.dev_status.cpu()[0]) == 0
    for name in ("U", "S", "V"):
        assert torch.equal(getattr(plain, name), getattr(comp, name))
    assert torch.equal(plain.U_q.codes, comp.U_q.codes) and torch.equal(plain.V_q.codes, comp.V_q.codes)
    A64 = d["W"].f64()
    Uq, Vq = read_fp4(comp.U_q), read_fp4(comp.V_q)
    S = comp.S.cpu().numpy().astype(np.float64)
    Rc = split.compensated_residual(A64, Uq, S, Vq)
    R = comp.R_f32.cpu().numpy()
    assert rel_fro(R, Rc) < TOL
    assert_fp4_equal(comp.R_rows, fp4.quantize(R, fmt, 1), check_linear=False)
    assert_fp4_equal(comp.R_cols, fp4.quantize(R, fmt, 0), check_linear=False)
    low = (Uq.dequantize().T * S) @ Vq.dequantize()
    err_c = rel_fro(low + read_fp4(comp.R_rows).dequantize(), A64)
    err_p = rel_fro(low + read_fp4(plain.R_rows).dequantize(), A64)
    assert err_c < err_p


@pytest.mark.parametrize("q", [0, 1])
def test_split_wide_spectrum(q):
    # singular values over six decades: sigma_i = 10^(-6 i / 31) for the top
    # 32 and a tail from 1e-7 down (2^(-1/16) apart).  How far down the GPU
    # resolves sigma is set by its arithmetic, not by the core solver (the
    # float64 Gram eigen-decomposition resolves about sqrt(eps64) sigma_1):
    #  q = 0: the products that form Y, Q and Z (bf16 hi / lo parts on the
    #    tensor cores) carry a backward error of order 2^-16 |A|;
    #  q = 1: the first basis is orthonormalised from A^T A Omega directly,
    #    whose float64 Gram spans sigma^4, so directions below
    #    eps64^(1/4) sigma_1 ~ 1.2e-4 sigma_1 are lost to its rounding.
    # Each sigma_i then moves by at most that floor (Weyl's inequality) and
    # each singular vector turns by at most floor / gap_i (Wedin's theorem);
    # the test takes eps = 4 x 2^-16 sigma_1 (q = 0) and 2 x eps64^(1/4)
    # sigma_1 (q = 1).
    rng = np.random.default_rng(19)
    m, n, k, p = 384, 256, 32, 16
    Ul, _ = np.linalg.qr(rng.standard_normal((m, n)))
    Vr, _ = np.linalg.qr(rng.standard_normal((n, n)))
    s = np.r_[10.0 ** (-6.0 * np.arange(k) / (k - 1)), 1e-7 * 2.0 ** (-np.arange(n - k) / 16.0)]
    A = ((Ul * s) @ Vr.T).astype(np.float32)
    A64 = A.astype(np.float64)
    res = api.split(torch.from_numpy(A).cuda(), k, p, q, 3, "nv", tap=True)
    torch.cuda.synchronize()
    assert int(res.dev_status.cpu()[0]) == 0
    ref = split.split(A64, k, p, q, 3)
    U = res.U.cpu().numpy().astype(np.float64)
    S = res.S.cpu().numpy().astype(np.float64)
    V = res.V.cpu().numpy().astype(np.float64)
    R = res.R_f32.cpu().numpy()
    assert all(np.all(np.isfinite(x)) for x in (U, S, V, R))
    assert np.all(S >= 0) and np.all(np.diff(S) <= 0)
    s_full = np.linalg.svd(A64, compute_uv=False)
    eps = (2.0 ** -14 if q == 0 else 2.0 * np.finfo(np.float64).eps ** 0.25) * s_full[0]
    dev = np.abs(S - ref["S"])
    assert dev.max() <= eps, (dev.max() / s_full[0], np.argmax(dev))
    # the well-resolved values (sigma_i >= 1e-2 sigma_1) to the split tolerance
    big = ref["S"] >= 1e-2 * s_full[0]
    assert np.max(dev[big] / ref["S"][big]) < 2e-3
    gap = np.minimum(s_full[:k] - s_full[1:k + 1], np.r_[np.inf, s_full[:k - 1] - s_full[1:k]])
    for j in range(k):
        tol = 2.0 * eps / gap[j]
        if tol > 0.1:
            continue
        for F, Fr in ((U, ref["U"]), (V, ref["V"])):
            e = min(np.linalg.norm(F[:, j] - Fr[:, j]), np.linalg.norm(F[:, j] + Fr[:, j]))
            assert e <= tol, (j, e, tol)
    L = (U * S) @ V.T
    assert rel_fro(L, (ref["U"] * ref["S"]) @ ref["V"].T) < TOL
    # the residual is the tail (|R| ~ 3e-7 |A|): the tap equals A - U S V^T of
    # the GPU's own factors to the products' rounding, relative to |A|
    assert np.linalg.norm(R.astype(np.float64) - (A64 - L)) / np.linalg.norm(A64) < 1e-5
    assert np.linalg.norm(R) / np.linalg.norm(A64) < 4 * eps / s_full[0] * np.sqrt(k)
    assert_fp4_equal(res.U_q, fp4.quantize(res.U.cpu().numpy(), "nv", 0), check_linear=False)
    assert_fp4_equal(res.V_q, fp4.quantize(res.V.cpu().numpy(), "nv", 0), check_linear=False)
    assert_fp4_equal(res.R_rows, fp4.quantize(R, "nv", 1), check_linear=False)
