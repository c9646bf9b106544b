"""Shared pytest setup: repo root on sys.path, the `gpu` marker, and helpers."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_sessionstart(session):
    """Build libcalibatt.so in-tree (nvcc, sm_100a) before the tests load it: a fresh
    checkout has none, and a library older than its sources would test old code.  The
    build skips itself when the library is up to date.  Without nvcc the oracle and format
    tests still run; the tests that load the library then report it missing."""
    from calibrated_block_sparse_calib_b200 import build
    try:
        build.build()
    except RuntimeError as e:
        sys.stderr.write(f"libcalibatt.so not built: {e}\n")


def to64(t):
    """bf16/fp32 torch tensor or array -> float64 numpy (exact upcast)."""
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return t.detach().to("cpu", torch.float32).numpy().astype(np.float64)
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(t, np.float64)


@pytest.fixture(scope="session")
def tiny_inputs():
    from calibrated_block_sparse_calib_b200 import synth
    wl = synth.WORKLOADS["tiny"]
    qkv = [synth.make_qkv(wl, input_idx=d) for d in range(wl.extra["n_calib"])]
    return wl, qkv
