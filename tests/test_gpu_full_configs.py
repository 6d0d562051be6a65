"""GPU parity at the full sizes of the workloads other than the timed layer.

Each workload runs through the library at its full size.  The oracle then
computes what it can afford one piece at a time: the split's singular values
in full, the rank-k part and the residual on sampled rows, the FP4 codes and
scales of the sampled rows (bit-exact, with the tensor maximum of the whole
residual for NVFP4), and the products on sampled output rows against the
float64 product of the GPU's own dequantized operands.  Tolerances are those
of the split (1e-3) and of the products (2e-3)."""
import numpy as np
import pytest
import torch

from oracle import averis, fp4, gemm, sketch, split
from spectral_domain_quantization_b200 import api, inputs

from gpu_helpers import read_fp4, rel_fro, to_device

pytestmark = pytest.mark.gpu

TOL_SPLIT = 1e-3
TOL_GEMM = 2e-3


def _rows(m, count, seed):
    return np.sort(np.random.default_rng(seed).choice(m, count, replace=False))


def _check_split_rows(A64, res, ref, rows, subspace=True):
    """S in full; the residual's energy; L and R on sampled rows (only where
    the top-k subspace is well determined: a matrix with a flat spectrum,
    like an iid Gaussian activation, has no unique top-k subspace, so there
    the invariant checks stand in); the blocks-along-n FP4 residual."""
    assert int(res.dev_status.cpu()[0]) == 0
    U = res.U.cpu().numpy().astype(np.float64)
    S = res.S.cpu().numpy().astype(np.float64)
    V = res.V.cpu().numpy().astype(np.float64)
    assert rel_fro(S, ref["S"]) < TOL_SPLIT
    L_rows = (U[rows] * S) @ V.T
    R = res.R_f32.cpu().numpy()
    r_energy = np.linalg.norm(R.astype(np.float64))
    assert abs(r_energy - np.linalg.norm(ref["R"])) / np.linalg.norm(ref["R"]) < TOL_SPLIT
    if subspace:
        Lref_rows = (ref["U"][rows] * ref["S"]) @ ref["V"].T
        assert rel_fro(L_rows, Lref_rows) < TOL_SPLIT
        assert rel_fro(R[rows], ref["R"][rows]) < TOL_SPLIT
    assert rel_fro(R[rows].astype(np.float64), A64[rows] - L_rows) < 1e-5
    if res.R_rows is not None:
        fmt = api.FMT_NAME[res.R_rows.fmt]
        amax = np.float32(np.abs(R).max()) if fmt == "nv" else None
        want = fp4.quantize(np.ascontiguousarray(R[rows]), fmt, 1, tensor_amax=amax)
        got = read_fp4(res.R_rows)
        assert np.array_equal(got.codes[rows], want.codes)
        assert np.array_equal(got.scales[rows], want.scales)
    return R


def test_llama3_mlp_gate_projection_full_size():
    """W 4096 x 14336, X 16384 x 4096, dY 16384 x 14336, all split (k = 64,
    p = 16, q = 1, NVFP4); Y = X W, dX = dY W^T and dW = X^T dY."""
    d = inputs.make("llama3_8b_mlp", keys=("W", "X", "dY"))
    c = d["cfg"]
    M, K, N, k = c["M"], c["K"], c["N"], c["k"]
    args = (k, c["p"], c["q"], c["sketch_seed"], "nv")
    Ws = api.split(to_device(d["W"]), *args, rows=True, cols=True, tap=True)
    Xs = api.split(to_device(d["X"]), *args, rows=True, cols=True, tap=True)
    Ds = api.split(to_device(d["dY"]), *args, rows=True, cols=True, tap=True)
    torch.cuda.synchronize()
    for name, res, m in (("W", Ws, K), ("X", Xs, M), ("dY", Ds, M)):
        A64 = d[name].f64()
        ref = split.split(A64, k, c["p"], c["q"], c["sketch_seed"])
        _check_split_rows(A64, res, ref, _rows(m, 64, 7), subspace=name == "W")
        del A64, ref
    # products on sampled output rows, from the GPU's own FP4 operands
    def op(qr, P, F, S):
        return gemm.Operand(read_fp4(qr), k, read_fp4(P), read_fp4(F), S.cpu().numpy().astype(np.float64))
    y = api.linear_fwd(Xs.operand("left"), Ws.operand("right"), M, N, K)
    dX, dW = api.linear_bwd(Ds.operand("left"), api.Operand(Ws.R_rows, k, Ws.V_q, Ws.U_q, Ws.S),
                            api.Operand(Xs.R_cols, k, Xs.U_q, Xs.V_q, Xs.S), Ds.operand("right"), M, N, K)
    torch.cuda.synchronize()
    rows = _rows(M, 64, 8)
    want = gemm.gemm(op(Xs.R_rows, Xs.V_q, Xs.U_q, Xs.S), op(Ws.R_cols, Ws.U_q, Ws.V_q, Ws.S), rows=rows)
    assert rel_fro(y.cpu().numpy()[rows], want) < TOL_GEMM
    want = gemm.gemm(op(Ds.R_rows, Ds.V_q, Ds.U_q, Ds.S), op(Ws.R_rows, Ws.V_q, Ws.U_q, Ws.S), rows=rows)
    assert rel_fro(dX.cpu().numpy()[rows], want) < TOL_GEMM
    rows_k = _rows(K, 64, 9)
    want = gemm.gemm(op(Xs.R_cols, Xs.U_q, Xs.V_q, Xs.S), op(Ds.R_cols, Ds.U_q, Ds.V_q, Ds.S), rows=rows_k)
    assert rel_fro(dW.cpu().numpy()[rows_k], want) < TOL_GEMM


def test_sampled_split_full_size():
    """A 65536 x 4096 with a rank-32 spike; 2048 sampled rows, sparse-sign
    sketch (4 nonzeros), k = 32, p = 16, q = 0, MXFP4; Y = A W (W plain)."""
    d = inputs.make("sampled_65536")
    c = d["cfg"]
    M, K, N = c["M"], c["K"], c["N"]
    res = api.split(to_device(d["A"]), c["k"], c["p"], 0, c["sketch_seed"], "mx", sketch="sparse_sign", nnz=4,
                    sample_rows=c["sample_rows"], rows=True, cols=False, tap=True)
    torch.cuda.synchronize()
    assert np.array_equal(res.idx.cpu().numpy(), sketch.sample_rows(M, c["sample_rows"], c["sketch_seed"]))
    A64 = d["A"].f64()
    ref = split.split(A64, c["k"], c["p"], 0, c["sketch_seed"], kind="sparse_sign", nnz=4,
                      sample_rows=c["sample_rows"])
    # at full size the spike lies below the noise edge (its directions are not
    # well separated), so the subspace-invariant checks apply
    _check_split_rows(A64, res, ref, _rows(M, 64, 10), subspace=False)
    del A64, ref
    w32 = d["W"].f32()
    qw = api.quantize_fp4(torch.from_numpy(w32).cuda(), "mx", 0)   # outer N, inner K
    y = api.linear_fwd(res.operand("left"), api.Operand(qw), M, N, K)
    torch.cuda.synchronize()
    rows = _rows(M, 64, 11)
    left = gemm.Operand(read_fp4(res.R_rows), c["k"], read_fp4(res.V_q), read_fp4(res.U_q),
                        res.S.cpu().numpy().astype(np.float64))
    want = gemm.gemm(left, gemm.Operand(read_fp4(qw)), rows=rows)
    assert rel_fro(y.cpu().numpy()[rows], want) < TOL_GEMM


def test_averis_full_size():
    """X 32768 x 4096 = 1 mu^T + Z, dY 32768 x 4096: mean split of both,
    NVFP4; Y = X W on sampled rows."""
    d = inputs.make("averis_32768")
    c = d["cfg"]
    M, K, N = c["M"], c["K"], c["N"]
    ax = api.averis_split(to_device(d["X"]), "nv", tap=True)
    ady = api.averis_split(to_device(d["dY"]), "nv", tap=False)
    torch.cuda.synchronize()
    x32 = d["X"].f32()
    mu = ax.mean.cpu().numpy()
    mu_ref, _ = averis.split(x32.astype(np.float64))
    assert np.max(np.abs(mu - mu_ref) / np.maximum(np.abs(mu_ref), 1e-3)) < 1e-6
    r32 = ax.R_f32.cpu().numpy()
    rows = _rows(M, 64, 12)
    assert np.array_equal(r32[rows], averis.residual_f32(x32[rows], mu))
    amax = np.float32(averis.residual_amax_from_columns(x32, mu))
    assert amax == np.abs(r32).max()
    want = fp4.quantize(np.ascontiguousarray(r32[rows]), "nv", 1, tensor_amax=amax)
    got = read_fp4(ax.R_rows)
    assert np.array_equal(got.codes[rows], want.codes)
    assert np.array_equal(got.scales[rows], want.scales)
    my_ref, _ = averis.split(d["dY"].f64())
    my = ady.mean.cpu().numpy()
    assert np.max(np.abs(my - my_ref) / np.maximum(np.abs(my_ref), 1e-6)) < 1e-5
    qw = api.quantize_fp4(to_device(d["W"]), "nv", 0)
    y = api.linear_fwd(ax.left(), api.Operand(qw), M, N, K)
    torch.cuda.synchronize()
    want = gemm.gemm(gemm.Operand(read_fp4(ax.R_rows), 1, read_fp4(ax.mean_q), "ones", [1.0]),
                     gemm.Operand(read_fp4(qw)), rows=rows)
    assert rel_fro(y.cpu().numpy()[rows], want) < TOL_GEMM


def _op(k, qr, P, F, S):
    """oracle operand from the GPU's own FP4 tensors"""
    return gemm.Operand(read_fp4(qr), k, read_fp4(P), read_fp4(F), S.cpu().numpy().astype(np.float64))


def test_tiny_forward_product():
    """W fp32 256 x 256 (planted, k = 8, p = 8, q = 1, MXFP4) split, X fp32
    128 x 256 quantized along K: Y = X W against the oracle's product of the
    same FP4 operands, and against the oracle's own chain from the inputs."""
    d = inputs.make("tiny_256")
    c = d["cfg"]
    M, K, N, k = c["M"], c["K"], c["N"], c["k"]
    ws = api.split(to_device(d["W"]), k, c["p"], c["q"], c["sketch_seed"], "mx", rows=False, cols=True)
    qx = api.quantize_fp4(to_device(d["X"]), "mx", 1)
    y = api.linear_fwd(api.Operand(qx), ws.operand("right"), M, N, K)
    torch.cuda.synchronize()
    assert int(ws.dev_status.cpu()[0]) == 0
    want = gemm.gemm(gemm.Operand(read_fp4(qx)), _op(k, ws.R_cols, ws.U_q, ws.V_q, ws.S))
    assert rel_fro(y.cpu().numpy(), want) < TOL_GEMM
    # the oracle's own chain: its split, its quantization, its product
    W64 = d["W"].f64()
    ref = split.split(W64, k, c["p"], c["q"], c["sketch_seed"])
    rq = fp4.quantize(ref["R"].astype(np.float32), "mx", 0)
    uq = fp4.quantize(ref["U"].astype(np.float32), "mx", 0)
    vq = fp4.quantize(ref["V"].astype(np.float32), "mx", 0)
    chain = gemm.gemm(gemm.Operand(fp4.quantize(d["X"].f32(), "mx", 1)),
                      gemm.Operand(rq, k, uq, vq, ref["S"]))
    assert rel_fro(y.cpu().numpy(), chain) < 2e-2


def test_layer_benched_call_full_size():
    """The timed step at its full size: split W 4096 x 4096 (k = 64, p = 16,
    q = 1, NVFP4, residual along K, FP4 factors), quantize X 8192 x 4096 along
    K, Y = X W with bf16 output.  The bf16 output is the float32 output of the
    same product rounded once; the float32 output matches the oracle's product
    of the same FP4 operands on sampled rows."""
    d = inputs.make("layer_4096")
    c = d["cfg"]
    M, K, N, k = c["M"], c["K"], c["N"], c["k"]
    ws = api.split(to_device(d["W"]), k, c["p"], c["q"], c["sketch_seed"], "nv", rows=False, cols=True)
    qx = api.quantize_fp4(to_device(d["X"]), "nv", 1)
    y16 = api.linear_fwd(api.Operand(qx), ws.operand("right"), M, N, K, out_dtype=torch.bfloat16)
    y = api.linear_fwd(api.Operand(qx), ws.operand("right"), M, N, K)
    torch.cuda.synchronize()
    assert int(ws.dev_status.cpu()[0]) == 0
    assert torch.equal(y16, y.to(torch.bfloat16))
    rows = _rows(M, 64, 13)
    want = gemm.gemm(gemm.Operand(read_fp4(qx)), _op(k, ws.R_cols, ws.U_q, ws.V_q, ws.S), rows=rows)
    assert rel_fro(y.cpu().numpy()[rows], want) < TOL_GEMM


def test_averis_backward_full_size():
    """X, dY 32768 x 4096 mean-split (NVFP4) along both axes, W 4096 x 4096:
    dX = dY W^T (contraction over N) and dW = X^T dY (contraction over M) on
    sampled output rows."""
    d = inputs.make("averis_32768")
    c = d["cfg"]
    M, K, N = c["M"], c["K"], c["N"]
    ax = api.averis_split(to_device(d["X"]), "nv", rows=False, cols=True)
    ady = api.averis_split(to_device(d["dY"]), "nv", rows=True, cols=True)
    qw_n = api.quantize_fp4(to_device(d["W"]), "nv", 1)          # outer K, blocks along N
    dX, dW = api.linear_bwd(ady.left(), api.Operand(qw_n), ax.left_t(), ady.right_m(), M, N, K)
    torch.cuda.synchronize()
    assert int(ax.dev_status.cpu()[0]) == 0 and int(ady.dev_status.cpu()[0]) == 0
    rows = _rows(M, 64, 14)
    left = gemm.Operand(read_fp4(ady.R_rows), 1, read_fp4(ady.mean_q), "ones", [1.0])
    want = gemm.gemm(left, gemm.Operand(read_fp4(qw_n)), rows=rows)
    assert rel_fro(dX.cpu().numpy()[rows], want) < TOL_GEMM
    rows_k = _rows(K, 64, 15)
    left = gemm.Operand(read_fp4(ax.R_cols), 1, "ones", read_fp4(ax.mean_q), [1.0])
    right = gemm.Operand(read_fp4(ady.R_cols), 1, "ones", read_fp4(ady.mean_q), [1.0])
    want = gemm.gemm(left, right, rows=rows_k)
    assert rel_fro(dW.cpu().numpy()[rows_k], want) < TOL_GEMM


def test_llama3_mlp_down_projection_full_size():
    """Down projection: W 14336 x 4096, H 16384 x 14336, dY 16384 x 4096, all
    split (k = 64, p = 16, q = 1, NVFP4); Y = H W, dH = dY W^T, dW = H^T dY."""
    d = inputs.make("llama3_8b_mlp", keys=("W_down", "H", "dY_down"))
    c = d["cfg"]
    M, K, N, k = c["M"], c["N"], c["K"], c["k"]   # contraction over the 14336 hidden units
    args = (k, c["p"], c["q"], c["sketch_seed"], "nv")
    Ws = api.split(to_device(d["W_down"]), *args, rows=True, cols=True, tap=True)
    Hs = api.split(to_device(d["H"]), *args, rows=True, cols=True, tap=True)
    Ds = api.split(to_device(d["dY_down"]), *args, rows=True, cols=True, tap=True)
    torch.cuda.synchronize()
    for name, res, m in (("W_down", Ws, K), ("H", Hs, M), ("dY_down", Ds, M)):
        A64 = d[name].f64()
        ref = split.split(A64, k, c["p"], c["q"], c["sketch_seed"])
        _check_split_rows(A64, res, ref, _rows(m, 64, 16), subspace=name == "W_down")
        del A64, ref
    y = api.linear_fwd(Hs.operand("left"), Ws.operand("right"), M, N, K)
    dH, dW = api.linear_bwd(Ds.operand("left"), api.Operand(Ws.R_rows, k, Ws.V_q, Ws.U_q, Ws.S),
                            api.Operand(Hs.R_cols, k, Hs.U_q, Hs.V_q, Hs.S), Ds.operand("right"), M, N, K)
    torch.cuda.synchronize()
    rows = _rows(M, 64, 17)
    want = gemm.gemm(_op(k, Hs.R_rows, Hs.V_q, Hs.U_q, Hs.S), _op(k, Ws.R_cols, Ws.U_q, Ws.V_q, Ws.S), rows=rows)
    assert rel_fro(y.cpu().numpy()[rows], want) < TOL_GEMM
    want = gemm.gemm(_op(k, Ds.R_rows, Ds.V_q, Ds.U_q, Ds.S), _op(k, Ws.R_rows, Ws.V_q, Ws.U_q, Ws.S), rows=rows)
    assert rel_fro(dH.cpu().numpy()[rows], want) < TOL_GEMM
    rows_k = _rows(K, 64, 18)
    want = gemm.gemm(_op(k, Hs.R_cols, Hs.U_q, Hs.V_q, Hs.S), _op(k, Ds.R_cols, Ds.U_q, Ds.V_q, Ds.S), rows=rows_k)
    assert rel_fro(dW.cpu().numpy()[rows_k], want) < TOL_GEMM
