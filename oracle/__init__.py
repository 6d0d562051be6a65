"""CPU oracle for the spectral-split W4A4G4 linear layer (Metis) and the Averis
mean/residual split.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, obviously-correct
restatement of what the GPU library computes.  Only the test suite, the
``smoke()`` check in ``__graft_entry__`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import it.  The product path
(the C ABI and its Python binding) never imports, calls or links anything here,
and nothing here imports the product path: the two share no code.  The only
module both sides consume is the seeded input generator
``spectral_domain_quantization_b200.inputs``, which holds none of the method's
arithmetic.

Arithmetic conventions
----------------------
* Linear algebra (sketch products, QR, SVD, residual, GEMM) runs in float64
  through numpy/LAPACK.
* The FP4 quantizer runs in IEEE float32 (numpy float32 operations round to
  nearest even), in exactly the operation order documented in ``fp4.py``, so
  that codes and scales can be compared bit for bit with the GPU kernels when
  both are fed the same float32 input.

Sources followed (page title, section)
--------------------------------------
* "Metis: Training LLMs with FP4 Quantization" (arXiv 2509.00404v4 summary),
  abstract and "method details / technical framework": the spectrum is split
  into a dominant part and a long tail that are quantized independently; the
  decomposition uses sparse random sampling and random projection.
* SII open-source-week release on Metis, section 2.3 (block-wise quantization:
  one scale per block, set by the block maximum; Fig. 3) and section 2.4 item 1
  (spectral decomposition into dominant and long-tail parts, randomized
  dimension reduction; MXFP4 / NVFP4 named in the feature list).
* "Metis: Training Large Language Models with Advanced Low-Bit Quantization"
  (older abstract), item (i): spectral decomposition with random embedding.
* Retelling of arXiv 2603.10444 (mean bias in FP4 LLM training), Averis method
  paragraphs: column mean over all rows, subtract, quantize mean and residual
  separately, the same split on the output gradient in the backward pass.

Everything the pages leave open (sketch distribution, QR/SVD form, FP4 scale
rules, op order, sampling law) follows one stated reading, numbered R1, R2,
...; each function below names the reading it implements and states it.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, brute force, published test vectors or independent
formulations.
"""

from . import philox, sketch, fp4, split, gemm, averis, composite, mlp, spectral_lr  # noqa: F401
