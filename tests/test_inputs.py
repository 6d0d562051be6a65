"""The seeded input generators: determinism, shapes, bf16 rounding (checked
against torch's own float32 -> bfloat16 conversion)."""
import numpy as np
import torch

from spectral_domain_quantization_b200 import inputs


def test_bf16_bits_match_torch():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(200000) * 10.0 ** rng.integers(-8, 8, 200000)).astype(np.float32)
    ours = inputs.to_bf16_bits(x)
    theirs = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, theirs)
    back = inputs.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_generators_deterministic_and_shaped():
    a = inputs.make("tiny_256")
    b = inputs.make("tiny_256")
    assert np.array_equal(a["W"].data, b["W"].data)
    assert a["W"].shape == (256, 256) and a["X"].shape == (128, 256)
    small = inputs.make("layer_4096", scale=dict(M=192, K=256, N=320))
    assert small["W"].shape == (256, 320) and small["X"].shape == (192, 256)
    assert small["W"].data.dtype == np.uint16


def test_planted_spectrum_visible():
    w = inputs.make("tiny_256")["W"].f64()
    s = np.linalg.svd(w, compute_uv=False)
    # sigma_1 = 4 planted on top of a 0.02 * sqrt(256) * 2 = 0.64 noise edge
    assert 3.0 < s[0] < 5.5
    assert s[40] < 1.0


def test_averis_activation_has_mean():
    d = inputs.make("averis_32768", scale=dict(M=4096, K=256, N=128))
    x = d["X"].f64()
    mu = x.mean(axis=0)
    assert 3.5 < mu.std() < 6.5          # mu_j ~ N(0, 25)
    z = x - mu
    assert 0.9 < np.median(np.abs(z)) / 0.674 < 1.2
