"""libqgemv: B200-native (sm_100a) weight-only quantized GEMV for LLM decode.

The C library (``libqgemv.so``, C ABI in ``include/qgemv.h``) does all the
work; ``qgemv`` is its thin ctypes binding, ``sweep`` runs a decoder-shaped
weight sweep through it in a CUDA graph, and ``workloads`` holds the shapes
and the seeded synthetic inputs.
"""
from . import workloads  # noqa: F401  (no CUDA needed)

__all__ = ["workloads", "qgemv", "sweep", "build"]
