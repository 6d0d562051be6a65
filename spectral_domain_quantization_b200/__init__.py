"""B200-native spectral-split FP4 linear layer (Metis) and Averis split.

The compute path is the C ABI in ``include/metis.h``, implemented by CUDA
kernels for sm_100a in ``csrc/`` and built into ``libmetis_b200.so``.  The
Python binding (``api``) only marshals torch tensors into that ABI.  Import
``spectral_domain_quantization_b200.api`` to use it; importing this package
alone loads nothing.
"""

__all__ = ["api", "inputs"]
