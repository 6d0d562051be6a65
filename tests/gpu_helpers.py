"""Helpers for the GPU parity tests: move seeded inputs to the device and read
GPU FP4 outputs back into the oracle's representation."""
import numpy as np
import torch

from oracle import fp4
from spectral_domain_quantization_b200 import api, inputs


def to_device(mat, device="cuda"):
    """inputs.Matrix or float32 numpy array -> CUDA tensor (bf16 or f32)."""
    if isinstance(mat, inputs.Matrix):
        if mat.dtype == "bf16":
            return torch.from_numpy(mat.data.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(mat.data).to(device)
    return torch.from_numpy(np.ascontiguousarray(mat)).to(device)


def bf16_tensor(x32, device="cuda"):
    """float32 numpy -> (bf16 CUDA tensor, float32 numpy of the bf16 values)."""
    bits = inputs.to_bf16_bits(x32)
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(device)
    return t, inputs.bf16_bits_to_f32(bits)


def read_fp4(q):
    """api.QTensor -> oracle FP4Tensor (decoded from the stored bytes)."""
    fmt = api.FMT_NAME[q.fmt]
    ts = float(q.tensor_scale.cpu().numpy()[0]) if fmt == "nv" else None
    return fp4.from_storage(fmt, q.outer, q.inner, q.codes.cpu().numpy(), q.scales.cpu().numpy(), ts)


def assert_fp4_equal(q, ref, check_linear=True):
    """Bit-exact comparison of a GPU QTensor with an oracle FP4Tensor."""
    assert (q.outer, q.inner) == (ref.outer, ref.inner)
    got_packed = q.codes.cpu().numpy().reshape(q.outer, q.inner // 2)
    want_packed = ref.packed
    if not np.array_equal(got_packed, want_packed):
        bad = np.argwhere(got_packed != want_packed)
        i, j = bad[0]
        raise AssertionError(f"{len(bad)} code bytes differ; first at {i},{j}: "
                             f"gpu {got_packed[i, j]:#04x} oracle {want_packed[i, j]:#04x}")
    got_sc = q.scales.cpu().numpy()
    want_sc = ref.scales_tc
    if not np.array_equal(got_sc, want_sc):
        bad = np.flatnonzero(got_sc != want_sc)
        raise AssertionError(f"{len(bad)} scale bytes differ; first at {bad[0]}: "
                             f"gpu {got_sc[bad[0]]} oracle {want_sc[bad[0]]}")
    if check_linear and q.scales_linear is not None:
        assert np.array_equal(q.scales_linear.cpu().numpy().reshape(ref.scales.shape), ref.scales)
    if ref.fmt == "nv":
        assert np.float32(q.tensor_scale.cpu().numpy()[0]) == np.float32(ref.tensor_scale)


def rel_fro(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    d = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (d if d > 0 else 1.0)
