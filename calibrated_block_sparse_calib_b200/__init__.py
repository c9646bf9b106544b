"""calibrated_block_sparse_calib_b200: calibrated block-sparse attention for one B200.

The compute path lives in ``libcalibatt.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/calibatt.h``); ``ops`` is a thin ctypes binding over it and
``synth`` makes seeded synthetic inputs.  There is no CPU fallback: every call raises if
the shared library or a CUDA device is missing.
"""
from . import synth  # noqa: F401

__all__ = ["synth"]
