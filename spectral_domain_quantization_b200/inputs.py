"""Seeded synthetic inputs for the spectral-split FP4 linear layer.

This module holds none of the method's arithmetic: it only draws matrices with
the shapes and spectra of the workloads the library is measured on, so that the
CPU oracle and the GPU path can be fed identical bytes.  It imports neither
side.

Recipe (all workloads): numpy PCG64 generators seeded per workload and per
matrix; "N(0, v)" means variance v; planted rank-one directions g_i, h_i are
iid N(0, 1/length) vectors; Gaussian arrays are drawn in float32 and rounded
to bfloat16 with round-to-nearest-even where the workload is bf16.

Workloads (the weight / activation / gradient shapes of an LLM linear layer):

* ``tiny_256``: W fp32 256x256 = sum_{i<=16} (4/i) g_i h_i^T + N(0, 0.02^2);
  X fp32 128x256 N(0,1); k=8, p=8, one power iteration, Gaussian sketch,
  seed 0; MXFP4; forward.
* ``layer_4096``: W bf16 4096x4096 with planted sigma_i = 8/i (i <= 256) plus
  N(0, 0.02^2); X bf16 8192x4096 N(0,1); k=64, p=16, one power iteration;
  NVFP4; forward.
* ``averis_32768``: X bf16 32768x4096 = 1 mu^T + Z, mu_j ~ N(0,25),
  Z ~ N(0,1) with 0.1% of entries multiplied by 20; W bf16 4096x4096
  N(0, 0.02^2) (plain NVFP4); dY bf16 32768x4096 N(0, 1e-4); forward and
  backward with the Averis split of X and dY.
* ``llama3_8b_mlp``: gate/up W 4096x14336 and down W 14336x4096 with planted
  sigma_i = 8/i (i <= 256) + N(0, 0.02^2); X bf16 16384x4096 N(0,1); down-proj
  input H 16384x14336 N(0,1); dY N(0, 1e-4); k=64, p=16, one power iteration;
  NVFP4 split of W, X and dY; forward, dX, dW.
* ``sampled_65536``: A bf16 65536x4096 with a planted rank-32 spike
  sigma_i = 50 i^-1.5 + N(0,1); 2048 sampled rows, sparse-sign sketch with 4
  nonzeros per input coordinate, k=32, p=16, no power iteration; MXFP4; GEMM
  with W bf16 4096x4096 N(0, 0.02^2) (plain MXFP4).
"""

import numpy as np

WORKLOADS = {
    "tiny_256": dict(M=128, K=256, N=256, k=8, p=8, q=1, fmt="mx", sketch="gaussian",
                     dtype="f32", seed=1001, sketch_seed=0),
    "layer_4096": dict(M=8192, K=4096, N=4096, k=64, p=16, q=1, fmt="nv", sketch="gaussian",
                       dtype="bf16", seed=1002, sketch_seed=0),
    "averis_32768": dict(M=32768, K=4096, N=4096, fmt="nv", dtype="bf16", seed=1003),
    "llama3_8b_mlp": dict(M=16384, K=4096, N=14336, k=64, p=16, q=1, fmt="nv",
                          sketch="gaussian", dtype="bf16", seed=1004, sketch_seed=0),
    "sampled_65536": dict(M=65536, K=4096, N=4096, k=32, p=16, q=0, fmt="mx",
                          sketch="sparse_sign", nnz=4, sample_rows=2048, dtype="bf16",
                          seed=1005, sketch_seed=0),
}


# --------------------------------------------------------------------------
# bfloat16 helpers (storage only)
# --------------------------------------------------------------------------

def to_bf16_bits(x):
    """float32 array -> uint16 bfloat16 bit patterns, round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    bias = np.uint64(0x7FFF) + ((bits >> np.uint64(16)) & np.uint64(1))
    return ((bits + bias) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(b):
    """uint16 bfloat16 bit patterns -> float32 values (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


class Matrix:
    """A generated matrix: ``bits`` (uint16 bf16 patterns) or ``f32`` data."""

    def __init__(self, data, dtype):
        self.dtype = dtype
        self.data = data

    @property
    def shape(self):
        return self.data.shape

    def f32(self):
        return bf16_bits_to_f32(self.data) if self.dtype == "bf16" else self.data

    def f64(self):
        return self.f32().astype(np.float64)


def _rng(seed, stream):
    return np.random.Generator(np.random.PCG64([int(seed), int(stream)]))


def _as(x, dtype):
    x = np.ascontiguousarray(x, dtype=np.float32)
    return Matrix(to_bf16_bits(x) if dtype == "bf16" else x, dtype)


def gaussian(shape, std, seed, stream, dtype="bf16"):
    x = _rng(seed, stream).standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return _as(x, dtype)


def planted(m, n, sigmas, noise_std, seed, stream, dtype="bf16"):
    """sum_i sigma_i g_i h_i^T + N(0, noise_std^2), g_i ~ N(0, 1/m), h_i ~ N(0, 1/n)."""
    rng = _rng(seed, stream)
    r = len(sigmas)
    g = rng.standard_normal((m, r), dtype=np.float32) / np.float32(np.sqrt(m))
    h = rng.standard_normal((n, r), dtype=np.float32) / np.float32(np.sqrt(n))
    x = (g * np.asarray(sigmas, dtype=np.float32)) @ h.T
    x += rng.standard_normal((m, n), dtype=np.float32) * np.float32(noise_std)
    return _as(x, dtype)


def averis_activation(m, n, seed, stream, dtype="bf16"):
    """1 mu^T + Z with mu_j ~ N(0, 25), Z ~ N(0,1), 0.1% of Z times 20."""
    rng = _rng(seed, stream)
    mu = rng.standard_normal(n, dtype=np.float32) * np.float32(5.0)
    z = rng.standard_normal((m, n), dtype=np.float32)
    mask = rng.random((m, n), dtype=np.float32) < np.float32(0.001)
    z[mask] *= np.float32(20.0)
    z += mu[None, :]
    return _as(z, dtype)


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------

def make(name, scale=None, keys=None):
    """Generate a workload's inputs.  ``scale`` optionally overrides sizes
    (dict of M/K/N) to get a smaller case with the same recipe; ``keys``
    optionally limits the matrices generated (each matrix has its own seeded
    stream, so the selection does not change their values)."""
    cfg = dict(WORKLOADS[name])
    if scale:
        cfg.update(scale)
    s = cfg["seed"]
    M, K, N = cfg["M"], cfg["K"], cfg["N"]
    if name == "tiny_256":
        gen = {"W": lambda: planted(K, N, [4.0 / i for i in range(1, 17)], 0.02, s, 1, "f32"),
               "X": lambda: gaussian((M, K), 1.0, s, 2, "f32")}
    elif name == "layer_4096":
        gen = {"W": lambda: planted(K, N, [8.0 / i for i in range(1, 257)], 0.02, s, 1),
               "X": lambda: gaussian((M, K), 1.0, s, 2)}
    elif name == "averis_32768":
        gen = {"X": lambda: averis_activation(M, K, s, 1),
               "W": lambda: gaussian((K, N), 0.02, s, 2),
               "dY": lambda: gaussian((M, N), 0.01, s, 3)}
    elif name == "llama3_8b_mlp":
        sig = [8.0 / i for i in range(1, 257)]
        gen = {"W": lambda: planted(K, N, sig, 0.02, s, 1),          # gate / up projection
               "W_down": lambda: planted(N, K, sig, 0.02, s, 2),     # down projection
               "X": lambda: gaussian((M, K), 1.0, s, 3),
               "H": lambda: gaussian((M, N), 1.0, s, 4),
               "dY": lambda: gaussian((M, N), 0.01, s, 5),           # gradient of gate / up output
               "dY_down": lambda: gaussian((M, K), 0.01, s, 6)}      # gradient of down output
    elif name == "sampled_65536":
        gen = {"A": lambda: planted(M, K, [50.0 * i ** -1.5 for i in range(1, 33)], 1.0, s, 1),
               "W": lambda: gaussian((K, N), 0.02, s, 2)}
    else:
        raise KeyError(name)
    out = dict(cfg=cfg)
    for key, fn in gen.items():
        if keys is None or key in keys:
            out[key] = fn()
    return out
