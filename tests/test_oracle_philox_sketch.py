"""Pins for the oracle's random generators: Philox4x32-10, the Gaussian and
sparse-sign sketches, row sampling, bfloat16 rounding."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import philox, sketch
from spectral_domain_quantization_b200 import inputs


def _kat(golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "philox4x32_10_kat.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            w = [int(t, 16) for t in line.split()]
            rows.append((w[:4], w[4:6], w[6:]))
    return rows


def test_philox_known_answers(golden_dir):
    kat = _kat(golden_dir)
    assert len(kat) == 3
    for ctr, key, out in kat:
        got = philox.philox4x32_10(*ctr, *key)
        assert [int(g) for g in got] == out


def test_philox_vectorised_matches_scalar():
    c = np.arange(17, dtype=np.uint64) * 0x01020305
    vec = philox.philox4x32_10(c, 7, 3, 0, 0xDEADBEEF, 0x12345678)
    for i in range(17):
        sc = philox.philox4x32_10(int(c[i]), 7, 3, 0, 0xDEADBEEF, 0x12345678)
        assert [int(v[i]) for v in vec] == [int(s) for s in sc]


def test_seed_key_split():
    assert philox.seed_key(0x0123456789ABCDEF) == (0x89ABCDEF, 0x01234567)


def _bf16_exact(x):
    """Nearest bfloat16 by exhaustive rational search over neighbours."""
    if x == 0:
        return 0.0
    a = Fraction(abs(x))
    e = math.frexp(abs(x))[1] - 1
    cands = []
    for ee in (e - 1, e, e + 1):
        ee = max(ee, -126)
        q = Fraction(2) ** (ee - 7)
        lo = Fraction(0) if ee == -126 else Fraction(2) ** ee
        hi = Fraction(2) ** (ee + 1)
        base = int(a / q)
        for mm in range(base - 2, base + 3):
            v = mm * q
            if mm >= 0 and lo <= v <= hi:
                # parity of the stored significand: the value's own binade
                cands.append((abs(a - v), (v / (Fraction(2) ** (max(math.frexp(float(v))[1] - 1, -126) - 7))) % 2 if v else 0, v))
    cands.sort(key=lambda t: (t[0], t[1]))
    return math.copysign(float(cands[0][2]), x)


def test_round_to_bf16_brute_force():
    rng = np.random.default_rng(5)
    xs = list(rng.standard_normal(300) * 10.0 ** rng.integers(-30, 30, 300))
    xs += [1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2 ** -130 * 1.5, 3.0 * 2 ** -134, 0.0]
    got = sketch.round_to_bf16(np.array(xs))
    want = [_bf16_exact(float(x)) for x in xs]
    assert np.array_equal(got, np.array(want))
    assert sketch.round_to_bf16(np.array([1 + 2 ** -8]))[0] == 1.0
    assert sketch.round_to_bf16(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6


def test_round_to_bf16_matches_bit_route_on_f32():
    # float32 inputs: the integer round-to-nearest-even on the bit pattern is an
    # independent route to the same values
    rng = np.random.default_rng(6)
    x = (rng.standard_normal(100000) * 3).astype(np.float32)
    a = sketch.round_to_bf16(x.astype(np.float64))
    b = inputs.bf16_bits_to_f32(inputs.to_bf16_bits(x)).astype(np.float64)
    assert np.array_equal(a, b)


def test_gaussian_sketch_moments_and_determinism():
    om = sketch.gaussian_omega(4096, 80, 0)
    assert om.shape == (4096, 80)
    assert np.array_equal(om, sketch.round_to_bf16(om))      # bf16 values
    z = om.ravel()
    n = z.size
    assert abs(z.mean()) < 5 / math.sqrt(n)
    assert abs(z.var() - 1) < 5 * math.sqrt(2 / n) + 2e-3    # bf16 rounding adds ~1e-5
    kurt = np.mean(z ** 4) / np.mean(z ** 2) ** 2
    assert abs(kurt - 3) < 5 * math.sqrt(24 / n) + 1e-2
    # even / odd columns (cos / sin of the same pair) are uncorrelated
    c = np.corrcoef(om[:, 0::2].ravel(), om[:, 1::2].ravel())[0, 1]
    assert abs(c) < 5 / math.sqrt(n / 2)
    assert np.array_equal(om, sketch.gaussian_omega(4096, 80, 0))
    assert not np.array_equal(om, sketch.gaussian_omega(4096, 80, 1))


def test_gaussian_sketch_ks():
    from scipy import stats
    om = sketch.gaussian_omega(2048, 64, 123).ravel()
    # bf16 rounding perturbs values by <= 2**-9 relative: KS distance stays tiny
    d = stats.kstest(om, "norm").statistic
    assert d < 1.63 / math.sqrt(om.size) + 3e-3


def test_gaussian_sketch_box_muller_pairs():
    # entries 2c and 2c+1 of a row come from one Philox block: r*cos, r*sin
    n, l, seed = 64, 16, 9
    om = sketch.gaussian_omega(n, l, seed)
    k0, k1 = philox.seed_key(seed)
    for i in (0, 5, 63):
        for c in range(l // 2):
            x0, x1, _, _ = philox.philox4x32_10(c, i, philox.STREAM_OMEGA, 0, k0, k1)
            u1 = (int(x0) + 1) / 2 ** 32
            r2 = -2 * math.log(u1)
            got = om[i, 2 * c] ** 2 + om[i, 2 * c + 1] ** 2
            assert abs(got - r2) <= 2 * 2 ** -7 * r2 + 1e-30


def test_gaussian_sketch_box_muller_angle():
    # the angle of the pair (even entry, odd entry) is 2 pi u2 with u2 from
    # the raw word x1: the even entry is r cos(theta) and the odd r sin(theta).
    # bf16 rounding moves each entry by at most 2**-9 of r, so the angle by at
    # most 2**-8; swapped cos / sin, u2 from another word, theta = pi u2 or a
    # flipped sign would all miss by far more on most pairs.
    n, l, seed = 96, 32, 4
    om = sketch.gaussian_omega(n, l, seed)
    k0, k1 = philox.seed_key(seed)
    checked = 0
    for i in range(n):
        for c in range(l // 2):
            x0, x1, _, _ = philox.philox4x32_10(c, i, philox.STREAM_OMEGA, 0, k0, k1)
            r = math.sqrt(-2 * math.log((int(x0) + 1) / 2 ** 32))
            if r < 1e-3:
                continue
            theta = 2 * math.pi * (int(x1) / 2 ** 32)
            got = math.atan2(om[i, 2 * c + 1], om[i, 2 * c])
            diff = (got - theta + math.pi) % (2 * math.pi) - math.pi
            assert abs(diff) <= 2 ** -8 + 1e-12, (i, c, got, theta)
            checked += 1
    assert checked > 0.99 * n * (l // 2)


def test_sparse_sign_structure():
    n, l, nnz = 4096, 48, 4
    om = sketch.sparse_sign_omega(n, l, nnz, 0)
    assert set(np.unique(om)) <= {-1.0, 0.0, 1.0}
    assert np.all(np.count_nonzero(om, axis=1) == nnz)
    # column usage ~ uniform: chi-square with l-1 dof
    counts = np.count_nonzero(om, axis=0)
    expect = n * nnz / l
    chi2 = np.sum((counts - expect) ** 2 / expect)
    assert chi2 < l + 6 * math.sqrt(2 * l)
    # signs balanced
    s = om[om != 0]
    assert abs(s.mean()) < 5 / math.sqrt(s.size)
    assert np.array_equal(om, sketch.sparse_sign_omega(n, l, nnz, 0))


def test_sparse_sign_reference_draw():
    # re-derive row 0 by hand from the Philox stream
    n, l, nnz, seed = 8, 5, 4, 77
    om = sketch.sparse_sign_omega(n, l, nnz, seed)
    k0, k1 = philox.seed_key(seed)
    for i in range(n):
        want = {}
        t = 0
        while len(want) < nnz:
            w = [int(v) for v in philox.philox4x32_10(t, i, philox.STREAM_SPARSE, 0, k0, k1)]
            for a, b in ((w[0], w[1]), (w[2], w[3])):
                col = int(Fraction(a * l, 2 ** 32))
                if len(want) < nnz and col not in want:
                    want[col] = -1.0 if b >= 2 ** 31 else 1.0
            t += 1
        row = np.zeros(l)
        for col, v in want.items():
            row[col] = v
        assert np.array_equal(om[i], row)


def test_sample_rows_brute_force():
    m, s, seed = 300, 37, 11
    idx = sketch.sample_rows(m, s, seed)
    k0, k1 = philox.seed_key(seed)
    keys = []
    for r in range(m):
        x0, x1, _, _ = philox.philox4x32_10(r, 0, philox.STREAM_SAMPLE, 0, k0, k1)
        keys.append(((int(x1) << 32) | int(x0), r))
    want = sorted(r for _, r in sorted(keys)[:s])
    assert list(idx) == want
    assert np.all(np.diff(idx) > 0)


def test_sample_rows_uniform_inclusion():
    m, s = 64, 16
    hits = np.zeros(m)
    trials = 400
    for seed in range(trials):
        hits[sketch.sample_rows(m, s, seed)] += 1
    p = s / m
    expect = trials * p
    sd = math.sqrt(trials * p * (1 - p))
    assert np.all(np.abs(hits - expect) < 5 * sd)
