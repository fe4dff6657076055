"""ECASQ on B200: entropy-constrained adaptive stochastic quantization.

The solver runs in hand-written sm_100a CUDA kernels behind the C ABI declared
in include/ecasq.h (library libecasq.so in this package). This package holds
the thin ctypes binding (ecasq.py) and the seeded input generators
(workloads.py). There is no CPU fallback: the first call into the binding
raises if the CUDA library is missing.
"""
__all__ = ["ecasq", "workloads"]
