"""B200 (sm_100a) implementation of the STEPQuant quantized gated Delta-rule decode step.

The product is libstepq.so (C ABI in include/stepq.h); ``stepq`` is its thin ctypes
binding and ``workloads`` draws seeded synthetic inputs.
"""
from . import stepq, workloads  # noqa: F401
