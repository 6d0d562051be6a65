"""Pins for the oracle's FP4 quantizer (E2M1 / E4M3 / E8M0 codecs, MXFP4 and
NVFP4 block quantization, storage layouts).  Every check uses a formulation
independent of ``oracle/fp4.py``: brute-force nearest-value search, exact
rationals, spec constants, reshape-based layouts, invariants."""
import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import fp4

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def brute_e2m1(q):
    """Nearest E2M1 magnitude by exhaustive distance, ties to the even code."""
    # magnitudes above 8 are nearest to 6 whatever they are; clamping keeps the
    # differences below exact in float64
    a = np.minimum(np.abs(q.astype(np.float64)), 8.0)
    d = np.abs(a[:, None] - np.array(E2M1)[None, :])
    dmin = d.min(axis=1, keepdims=True)
    cand = d == dmin
    even = cand & (np.arange(8)[None, :] % 2 == 0)
    code = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    return (code | (np.signbit(q).astype(np.int64) << 3)).astype(np.uint8)


def test_e2m1_round_trip_every_code():
    for c in range(16):
        v = fp4.e2m1_decode(np.array([c], np.uint8))
        v32 = np.array([-0.0 if c == 8 else v[0]], np.float32)
        assert fp4.e2m1_encode(v32)[0] == c
    assert fp4.e2m1_decode(np.arange(8, dtype=np.uint8)).tolist() == E2M1


def test_e2m1_ties_and_saturation():
    q = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 1e30, -0.1, -0.25, -5.0], np.float32)
    want = [0, 2, 2, 4, 4, 6, 6, 7, 7, 8, 8, 8 | 6]
    assert fp4.e2m1_encode(q).tolist() == want


def test_e2m1_dense_sweep_vs_brute_force():
    # every float32 with exponent in [-4, 3] (all of the interesting range)
    # plus random bit patterns over the whole finite range
    exps = np.arange(-4, 4) + 127
    mant = np.arange(0, 1 << 23, 7, dtype=np.uint32)
    bits = ((exps[:, None].astype(np.uint32) << 23) | mant[None, :]).ravel()
    rng = np.random.default_rng(0)
    rb = rng.integers(0, 0xFF000000, 2_000_000, dtype=np.uint64).astype(np.uint32)
    rb = rb[((rb >> 23) & 0xFF) != 0xFF]
    allbits = np.concatenate([bits, bits | np.uint32(0x80000000), rb])
    q = allbits.view(np.float32)
    assert np.array_equal(fp4.e2m1_encode(q), brute_e2m1(q))


def test_e2m1_exhaustive_near_midpoints():
    mids = [(E2M1[i] + E2M1[i + 1]) / 2 for i in range(7)] + [6.0]
    vals = []
    for m in mids:
        x = np.float32(m)
        for k in range(-3, 4):
            vals.append(np.nextafter(x, np.float32(np.inf if k > 0 else -np.inf)) if k else x)
            x2 = x
            for _ in range(abs(k)):
                x2 = np.nextafter(x2, np.float32(np.inf if k > 0 else -np.inf))
            vals.append(x2)
    q = np.array(vals, np.float32)
    q = np.concatenate([q, -q])
    assert np.array_equal(fp4.e2m1_encode(q), brute_e2m1(q))


E4M3_VALUES = fp4.e4m3_decode(np.arange(127))


def brute_e4m3(t):
    t = np.asarray(t, np.float64)
    d = np.abs(t[:, None] - E4M3_VALUES[None, :])
    dmin = d.min(axis=1, keepdims=True)
    cand = d == dmin
    even = cand & (np.arange(127)[None, :] % 2 == 0)
    return np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1)).astype(np.uint8)


def test_e4m3_decode_spec_points():
    # OCP 8-bit floating point spec, E4M3: bias 7, max normal 448, min normal 2**-6,
    # min subnormal 2**-9, 0x7F is NaN
    assert fp4.e4m3_decode(np.array([0x7E]))[0] == 448.0
    assert fp4.e4m3_decode(np.array([0x08]))[0] == 2.0 ** -6
    assert fp4.e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9
    assert fp4.e4m3_decode(np.array([0x38]))[0] == 1.0
    assert fp4.e4m3_decode(np.array([0x07]))[0] == 7 * 2.0 ** -9
    assert np.isnan(fp4.e4m3_decode(np.array([0x7F]))[0])
    assert np.all(np.diff(E4M3_VALUES) > 0)


def test_e4m3_encode_vs_brute_force():
    rng = np.random.default_rng(1)
    mids = (E4M3_VALUES[1:] + E4M3_VALUES[:-1]) / 2
    t = np.concatenate([
        E4M3_VALUES, mids, np.nextafter(mids, 0), np.nextafter(mids, 1000),
        rng.random(20000) * 500, np.exp(rng.uniform(-25, 7, 20000)),
        [448.0, 463.9, 464.0, 470.0, 1e6, 0.0, 2.0 ** -10, 2.0 ** -10 * 1.0001],
    ])
    assert np.array_equal(fp4.e4m3_encode(t), brute_e4m3(t))


def test_e8m0_closed_form():
    assert fp4.e8m0_decode(np.array([127]))[0] == 1.0
    assert fp4.e8m0_decode(np.array([0]))[0] == 2.0 ** -127
    assert fp4.e8m0_decode(np.array([254]))[0] == 2.0 ** 127
    assert np.isnan(fp4.e8m0_decode(np.array([255]))[0])


def _blocks(rng, rows, cols, spread=6):
    x = rng.standard_normal((rows, cols)) * np.exp2(rng.integers(-spread, spread, (rows, 1)))
    return x.astype(np.float32)


@pytest.mark.parametrize("axis", [0, 1])
def test_mx_scale_closed_form_and_invariants(axis):
    rng = np.random.default_rng(2)
    X = _blocks(rng, 64, 256)
    X[3, :32] = 0.0                                        # a zero block (axis=1)
    t = fp4.quantize(X, "mx", axis=axis)
    Z = X if axis == 1 else X.T
    blocks = Z.reshape(t.outer, t.inner // 32, 32).astype(np.float64)
    amax = np.abs(blocks).max(axis=2)
    for (i, j), a in np.ndenumerate(amax):
        if a == 0:
            assert t.scales[i, j] == 0
            assert np.all(t.codes[i, 32 * j:32 * j + 32] == 0)
            continue
        # OCP MX v1.0: shared exponent = floor(log2(amax)) - emax(E2M1), emax = 2
        se = math.frexp(a)[1] - 1 - 2
        assert t.scales[i, j] == se + 127
        codes = t.codes[i, 32 * j:32 * j + 32]
        # the block maximum lands on 4 or 6 (codes 6/7 magnitude)
        k = int(np.argmax(np.abs(blocks[i, j])))
        assert (codes[k] & 7) in (6, 7)
        # every element is within half a grid step of its dequantized value
        deq = fp4.e2m1_decode(codes) * 2.0 ** se
        q = blocks[i, j] / 2.0 ** se
        for x, qq, dv in zip(blocks[i, j], q, deq):
            aq = abs(qq)
            if aq > 6:
                assert abs(dv) == 6 * 2.0 ** se
                continue
            hi = min(v for v in E2M1 if v >= aq)
            lo = max(v for v in E2M1 if v <= aq)
            assert abs(aq - abs(dv) / 2.0 ** se) <= (hi - lo) / 2 + 1e-12


def test_mx_exact_values_round_trip():
    # blocks made of E2M1 values times a power of two whose max is 6 or 4
    rng = np.random.default_rng(3)
    vals = np.array(E2M1 + [-v for v in E2M1[1:]])
    X = rng.choice(vals, (16, 64))
    X[:, 0] = 6.0
    X[:, 32] = -4.0
    scale = np.exp2(rng.integers(-20, 20, (16, 1)))
    X = (X * scale).astype(np.float32)
    t = fp4.quantize(X, "mx")
    assert np.array_equal(t.dequantize(), X.astype(np.float64))


def test_nv_two_level_scale():
    rng = np.random.default_rng(4)
    X = _blocks(rng, 32, 128, spread=3)
    t = fp4.quantize(X, "nv")
    alpha = np.float32(np.abs(X).max())
    assert t.tensor_scale == np.float32(alpha / np.float32(2688.0))
    # the block holding the global maximum gets scale 448 and its max code 6
    i, j = np.unravel_index(np.argmax(np.abs(X)), X.shape)
    assert fp4.e4m3_decode(t.scales[i, j // 16]) == 448.0
    assert (t.codes[i, j] & 7) == 7
    # dequantized block maxima are within the E4M3 rounding of the true maxima
    blocks = X.reshape(32, 8, 16).astype(np.float64)
    amax = np.abs(blocks).max(axis=2)
    bscale = fp4.e4m3_decode(t.scales) * float(t.tensor_scale)
    nz = amax > 0
    ratio = (amax[nz] / 6) / bscale[nz]
    assert np.all(np.abs(ratio - 1) < 2.0 ** -4 + 1e-6)


def test_nv_reference_arithmetic_one_block():
    # re-derive one block's codes with exact rationals and float32 rounding steps
    rng = np.random.default_rng(5)
    X = (rng.standard_normal((1, 32)) * 3).astype(np.float32)
    t = fp4.quantize(X, "nv")
    f32 = lambda v: float(np.float32(v))
    alpha = float(np.abs(X).max())
    s_t = f32(alpha / 2688.0)
    for b in range(2):
        blk = X[0, 16 * b:16 * b + 16].astype(np.float64)
        tval = f32(f32(float(np.abs(blk).max()) / s_t) / 6.0)
        d = float(E4M3_VALUES[brute_e4m3([tval])[0]])
        enc = f32(1.0 / f32(d * s_t))
        q = np.array([f32(x * enc) for x in blk], np.float32)
        assert np.array_equal(t.codes[0, 16 * b:16 * b + 16], brute_e2m1(q))


def test_quantize_is_sign_symmetric():
    rng = np.random.default_rng(6)
    X = _blocks(rng, 16, 64)
    for fmt in ("mx", "nv"):
        a = fp4.quantize(X, fmt)
        b = fp4.quantize(-X, fmt)
        assert np.array_equal(a.scales, b.scales)
        nz = (a.codes & 7) != 0
        assert np.array_equal(a.codes[nz] ^ 8, b.codes[nz])


def test_axis0_is_transpose():
    rng = np.random.default_rng(7)
    X = _blocks(rng, 96, 64)
    for fmt in ("mx", "nv"):
        a = fp4.quantize(X, fmt, axis=0)
        b = fp4.quantize(np.ascontiguousarray(X.T), fmt, axis=1)
        assert np.array_equal(a.codes, b.codes) and np.array_equal(a.scales, b.scales)


def test_pack_layout():
    codes = np.arange(32, dtype=np.uint8).reshape(2, 16) % 16
    p = fp4.pack_codes(codes)
    assert p[0, 0] == (codes[0, 0] | (codes[0, 1] << 4))
    assert np.array_equal(fp4.unpack_codes(p), codes)


@pytest.mark.parametrize("bs", [16, 32])
def test_tensor_core_scale_layout_vs_reshape(bs):
    outer, inner = 300, 1024 + 256
    rng = np.random.default_rng(8)
    s = rng.integers(1, 255, (outer, inner // bs)).astype(np.uint8)
    flat = fp4.swizzle_scales(s, bs)
    # independent route: pad, view as [row-group][32][4][col-chunk][4], reorder
    R = -(-outer // 128) * 128
    C = -(-(inner // bs) // (256 // bs)) * (256 // bs)
    P = np.zeros((R, C), np.uint8)
    P[:outer, :inner // bs] = s
    # row r = 128*g + 32*h + w, col c = 4*j + b  ->  [g][j][w][h][b]
    V = P.reshape(R // 128, 4, 32, C // 4, 4).transpose(0, 3, 2, 1, 4)
    assert np.array_equal(flat, V.ravel())
    assert np.array_equal(fp4.unswizzle_scales(flat, outer, inner, bs), s)


def test_from_storage_round_trip():
    rng = np.random.default_rng(9)
    X = _blocks(rng, 130, 512)
    for fmt in ("mx", "nv"):
        t = fp4.quantize(X, fmt)
        u = fp4.from_storage(fmt, t.outer, t.inner, t.packed, t.scales_tc, t.tensor_scale)
        assert np.array_equal(u.dequantize(), t.dequantize())


def test_dequantize_exact_rational():
    rng = np.random.default_rng(10)
    X = _blocks(rng, 4, 64)
    for fmt in ("mx", "nv"):
        t = fp4.quantize(X, fmt)
        d = t.dequantize()
        for i in range(4):
            for j in range(0, 64, 7):
                c = int(t.codes[i, j])
                v = Fraction(E2M1[c & 7]) * (-1 if c & 8 else 1)
                if fmt == "mx":
                    s = Fraction(2) ** (int(t.scales[i, j // 32]) - 127)
                else:
                    s = Fraction(float(E4M3_VALUES[t.scales[i, j // 16]])) * Fraction(float(t.tensor_scale))
                assert Fraction(d[i, j]) == v * s
