"""The synthetic W4A4G4 MLP training step on the GPU (spectral_domain_quantization_b200.mlp,
reading R31) against the oracle (oracle/mlp.py).

Every product of a step is held to the oracle's float64 product of the very
FP4 operands the library used (2e-3, the product tolerance).  The whole step
is compared with the oracle's own chain under the same policy: under "fp4"
the two quantize the same float32 values up to the float32 rounding of the
intermediate activations, so the gradients agree to the product tolerance;
under "metis" the splits agree to 1e-3 and their FP4 codes may differ where
a factor entry straddles a rounding boundary, so the gradients are held to
the looser bound stated there.  A short training run under both policies
must reduce the loss as the oracle's float64 run does (the loss curves are
printed)."""
import numpy as np
import pytest
import torch

from oracle import gemm
from oracle import mlp as omlp
from spectral_domain_quantization_b200 import mlp

from gpu_helpers import read_fp4, rel_fro

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(np.float32(a))).cuda()


def _oracle_operand(op):
    R = read_fp4(op.R)
    if op.k == 0:
        return gemm.Operand(R)
    return gemm.Operand(R, op.k, read_fp4(op.P), read_fp4(op.F), op.S.cpu().numpy().astype(np.float64))


@pytest.mark.parametrize("kind", ["fp4", "metis"])
@pytest.mark.parametrize("fmt", ["nv", "mx"])
def test_training_step(kind, fmt):
    X, T, (W1, W2) = omlp.problem()
    loss, (dW1, dW2), record = mlp.step((_dev(W1), _dev(W2)), _dev(X), _dev(T), mlp.Policy(kind, fmt))
    torch.cuda.synchronize()
    assert [r[0] for r in record] == ["fwd", "fwd", "dx", "dw", "dw"]
    for name, left, right, out in record:
        want = gemm.gemm(_oracle_operand(left), _oracle_operand(right))
        assert rel_fro(out.cpu().numpy(), want) < 2e-3, name
    ref_loss, (r1, r2) = omlp.loss_and_grads((W1, W2), X, T, omlp.Policy(kind, fmt))
    e1, e2 = rel_fro(dW1.cpu().numpy(), r1), rel_fro(dW2.cpu().numpy(), r2)
    print(f"mlp step {kind} {fmt}: loss {loss:.6f} (oracle {ref_loss:.6f}), dW1 {e1:.2e}, dW2 {e2:.2e}")
    assert abs(loss - ref_loss) <= 1e-3 * ref_loss
    tol = 2e-3 if kind == "fp4" else 2e-2
    assert e1 < tol and e2 < tol


def test_training_curves():
    X, T, params = omlp.problem()
    steps, lr = 60, 1.0
    ref, _ = omlp.train(params, X, T, omlp.Policy("exact"), lr, steps)
    for kind in ("fp4", "metis"):
        for fmt in ("nv", "mx"):
            losses, _ = mlp.train((_dev(params[0]), _dev(params[1])), _dev(X), _dev(T), mlp.Policy(kind, fmt),
                                  lr, steps)
            losses = np.array(losses)
            print(f"mlp curve {kind} {fmt}: " + " ".join(f"{v:.4f}" for v in losses[::10]) +
                  f" final {losses[-1]:.4f} (float64 {ref[-1]:.4f})")
            assert np.all(np.isfinite(losses))
            assert losses[-1] < 0.5 * losses[0]
            assert losses[-1] < 1.5 * ref[-1]
