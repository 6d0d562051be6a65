"""GPU parity of metis_quantize_fp4 against the oracle quantizer: codes,
tensor-core scales, linear scales and tensor scale bit-exact on identical
float32 inputs; inner sums within float32 summation error."""
import numpy as np
import pytest
import torch

from oracle import fp4
from spectral_domain_quantization_b200 import api, inputs

from gpu_helpers import assert_fp4_equal, bf16_tensor, rel_fro

pytestmark = pytest.mark.gpu


def _data(rows, cols, seed, spread=8):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)) * np.exp2(rng.integers(-spread, spread, (rows, 1)))
    x *= np.exp2(rng.integers(-3, 3, (1, cols)))
    x[rng.random((rows, cols)) < 0.01] *= 50.0
    return x.astype(np.float32)


def _run(x32, dtype, fmt, axis, sub=None, inner_sum=True):
    # rows must start on 16-byte boundaries: pad the leading dimension and
    # pass a column view when the width does not allow it
    rows, cols = x32.shape
    per16 = 8 if dtype == "bf16" else 4
    ld = -(-cols // per16) * per16
    xp = np.zeros((rows, ld), np.float32)
    xp[:, :cols] = x32
    if dtype == "bf16":
        Xp, xval = bf16_tensor(xp)
    else:
        Xp, xval = torch.from_numpy(xp).cuda(), xp
    X = Xp[:, :cols]
    xval = np.ascontiguousarray(xval[:, :cols])
    sub_t = None if sub is None else torch.from_numpy(sub).cuda()
    q = api.quantize_fp4(X, fmt, axis, sub_col=sub_t, linear=True, inner_sum=inner_sum)
    torch.cuda.synchronize()
    xin = xval if sub is None else (xval - sub[None, :]).astype(np.float32)
    ref = fp4.quantize(xin, fmt, axis)
    return q, ref


SHAPES = [(96, 320), (300, 1024 + 32), (1, 64), (129, 96), (64, 4096)]


@pytest.mark.parametrize("fmt", ["mx", "nv"])
@pytest.mark.parametrize("axis", [0, 1])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", SHAPES)
def test_quantize_bit_exact(fmt, axis, dtype, shape):
    rows, cols = shape
    if axis == 0:
        rows, cols = cols, rows          # blocked dimension must be a multiple of 32
    x = _data(rows, cols, hash((fmt, axis, dtype, shape)) % 2 ** 31)
    q, ref = _run(x, dtype, fmt, axis)
    assert_fp4_equal(q, ref)
    got = q.inner_sum.cpu().numpy()
    assert rel_fro(got, ref.colsum()) < 1e-5


@pytest.mark.parametrize("fmt", ["mx", "nv"])
@pytest.mark.parametrize("axis", [0, 1])
def test_quantize_with_column_subtraction(fmt, axis):
    rows, cols = (256, 192) if axis == 1 else (192 + 64, 96)
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((rows, cols)) + rng.standard_normal(cols) * 5).astype(np.float32)
    mu = x.astype(np.float64).mean(axis=0).astype(np.float32)
    q, ref = _run(x, "bf16", fmt, axis, sub=mu)
    assert_fp4_equal(q, ref)


@pytest.mark.parametrize("fmt", ["mx", "nv"])
def test_quantize_edge_values(fmt):
    rows, cols = 64, 256
    x = _data(rows, cols, 11)
    x[0] = 0.0                                   # zero rows / blocks
    x[1, :32] = -0.0
    x[2] = 1e30                                  # huge
    x[3] = np.float32(1e-40)                     # subnormal
    x[4, ::2] = 6.0
    x[4, 1::2] = -0.2
    x[5] = np.float32(2.0) ** -126
    for axis in (0, 1):
        xx = x if axis == 1 else np.ascontiguousarray(x.T)
        q, ref = _run(xx, "f32", fmt, axis)
        assert_fp4_equal(q, ref)


def test_quantize_all_zero_nvfp4():
    x = np.zeros((32, 64), np.float32)
    q, ref = _run(x, "f32", "nv", 1)
    assert_fp4_equal(q, ref)
    assert float(q.tensor_scale.cpu()[0]) == 1.0


def test_e2m1_sweep_through_mx_blocks():
    # a block whose maximum is 6.0 has scale 2^0, so the other 31 elements are
    # encoded as-is: sweep float32 patterns of magnitude below 8
    exps = np.arange(-10, 3) + 127
    mant = np.arange(0, 1 << 23, 97, dtype=np.uint32)
    bits = ((exps[:, None].astype(np.uint32) << 23) | mant[None, :]).ravel()
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    near = np.concatenate([mids, np.nextafter(mids, 0), np.nextafter(mids, 9)])
    vals = np.concatenate([bits.view(np.float32), near])
    vals = np.concatenate([vals, -vals])
    nblk = -(-vals.size // 31)
    pad = np.zeros(nblk * 31, np.float32)
    pad[:vals.size] = vals
    x = np.concatenate([np.full((nblk, 1), 6.0, np.float32), pad.reshape(nblk, 31)], axis=1)
    rows = 1024
    nb = -(-nblk // rows)
    X = np.zeros((rows * nb, 32), np.float32)
    X[:nblk] = x
    X = np.ascontiguousarray(X.reshape(rows, nb * 32))
    q, ref = _run(X, "f32", "mx", 1, inner_sum=False)
    assert_fp4_equal(q, ref)


def test_e4m3_sweep_through_nv_scales():
    # tensor max 2688 makes s_t = 1, so each block's t is fl(amax / 6)
    e4 = fp4.e4m3_decode(np.arange(127))
    mids = (e4[1:] + e4[:-1]) / 2
    # (block maxima cannot exceed the tensor maximum, so t stays <= 448)
    t = np.concatenate([e4, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
                        np.linspace(0, 448, 4001)]).astype(np.float32)
    t = t[t <= 448]
    a = (t.astype(np.float64) * 6).astype(np.float32)
    nblk = a.size
    rows = -(-nblk // 32)
    X = np.zeros((rows * 32, 16), np.float32)    # one 16-element block per row of X
    X[:nblk, 0] = a
    X[0, 1] = 2688.0
    Y = np.ascontiguousarray(X.reshape(rows, 32 * 16))
    q, ref = _run(Y, "f32", "nv", 1, inner_sum=False)
    assert float(ref.tensor_scale) == 1.0
    assert_fp4_equal(q, ref)


@pytest.mark.parametrize("axis", [1, 0])
def test_quantize_full_size_activation(axis):
    # the 8192 x 4096 bf16 activation of the single-layer workload, NVFP4
    d = inputs.make("layer_4096")
    X = torch.from_numpy(d["X"].data.view(np.int16)).view(torch.bfloat16).cuda()
    q = api.quantize_fp4(X, "nv", axis)
    torch.cuda.synchronize()
    ref = fp4.quantize(d["X"].f32(), "nv", axis)
    assert_fp4_equal(q, ref)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("axis", [0, 1])
def test_quantize_strided_view(dtype, axis):
    # a column view of a wider matrix (leading dimension 320 > 256 columns):
    # the NVFP4 tensor maximum and the codes must ignore the columns outside
    # the view, which hold the largest values of the buffer
    rows, cols, ld = 224, 256, 320
    x = _data(rows, ld, 21)
    x[:, cols:] *= 1e3
    if dtype == "bf16":
        Xp, xval = bf16_tensor(x)
    else:
        Xp, xval = torch.from_numpy(x).cuda(), x
    q = api.quantize_fp4(Xp[:, :cols], "nv", axis, linear=True)
    torch.cuda.synchronize()
    ref = fp4.quantize(np.ascontiguousarray(xval[:, :cols]), "nv", axis)
    assert_fp4_equal(q, ref)
