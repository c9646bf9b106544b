"""Host-side checks of the C ABI (CPU only): the library loads and exports every
function include/calibatt.h declares, status strings, and argument validation that
rejects bad calls before any device work."""
import ctypes
import os
import re

import pytest

from calibrated_block_sparse_calib_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"^\s*(?:const\s+)?[\w]+\**\s+\**(\w+)\s*\(", src, flags=re.M))
    return names


def test_library_exports_every_declared_symbol():
    L = ops.lib()
    declared = _declared()
    assert {"sparse_attn_fwd", "sparse_attn_fwd_repeat", "calib_block_energy", "calib_select_mask"} <= declared
    for name in declared:
        assert hasattr(L, name), name
    assert declared <= set(ops._SIGS), "binding is missing a declared entry point"


def test_status_strings():
    assert ops.status_string(ops.CALIB_OK) == "CALIB_OK"
    assert ops.status_string(ops.CALIB_ERR_TIMEOUT) == "CALIB_ERR_TIMEOUT"


def test_anchor_count_host():
    assert ops.anchor_count(21, 45, 80, 0, 4) == 21 * 12 * 80
    assert ops.anchor_count(4, 8, 16, 0, 2) == 256
    assert ops.lib().calib_anchor_count(1, 1, 1, 0, 0) == -1


def test_invalid_arguments_rejected_before_device_work():
    L = ops.lib()
    null = ctypes.c_void_p(0)
    # null pointers
    assert L.calib_select_mask(null, 1, 1, 1, 0.9, null, null, null, null) == ops.CALIB_ERR_INVALID
    # tau outside (0, 1]
    fake = ctypes.c_void_p(256)
    assert L.calib_select_mask(fake, 1, 1, 1, 0.0, null, fake, null, null) == ops.CALIB_ERR_INVALID
    assert L.calib_select_mask(fake, 1, 1, 1, 1.5, null, fake, null, null) == ops.CALIB_ERR_INVALID
    # rho outside [0, 1]
    assert L.calib_aggregate_masks(fake, 1, 1, 1, 3, 3, 2, fake, null) == ops.CALIB_ERR_INVALID
    # block size, misalignment, missing list
    assert L.calib_block_energy(fake, fake, null, 1, 128, 128, 96, 0.1, null, 0, fake, 0, null) == \
        ops.CALIB_ERR_INVALID
    assert L.calib_block_energy(ctypes.c_void_p(258), fake, null, 1, 128, 128, 128, 0.1, null, 0, fake, 0,
                                null) == ops.CALIB_ERR_INVALID
    assert L.sparse_attn_fwd(fake, fake, fake, fake, null, 1, 128, 128, 0.1, None, 0, null) == ops.CALIB_ERR_INVALID
    bl = ops._BlockListC(1, 1, 1, 128, 256, 256, 0, 0)
    # head dim not supported
    assert L.sparse_attn_fwd(fake, fake, fake, fake, null, 1, 128, 96, 0.1, ctypes.byref(bl), 0, null) == \
        ops.CALIB_ERR_UNSUPPORTED
    # list shape mismatch (nq != ceil(N/B))
    bl2 = ops._BlockListC(1, 2, 2, 128, 256, 256, 0, 0)
    assert L.sparse_attn_fwd(fake, fake, fake, fake, null, 1, 128, 128, 0.1, ctypes.byref(bl2), 0, null) == \
        ops.CALIB_ERR_INVALID
    # negative scale
    assert L.sparse_attn_fwd(fake, fake, fake, fake, null, 1, 128, 128, -1.0, ctypes.byref(bl), 0, null) == \
        ops.CALIB_ERR_INVALID
    # unknown flag bits
    assert L.sparse_attn_fwd(fake, fake, fake, fake, null, 1, 128, 128, 0.1, ctypes.byref(bl), 6, null) == \
        ops.CALIB_ERR_INVALID
    # host-buffer attention: null host pointers, a chunk size below 1, then the device
    # buffers' checks (head dim, list shape)
    assert L.sparse_attn_fwd_host(null, fake, fake, fake, fake, fake, fake, fake, null, 1, 128, 128, 0.1,
                                  ctypes.byref(bl), 0, 1, null, null, null) == ops.CALIB_ERR_INVALID
    assert L.sparse_attn_fwd_host(fake, fake, fake, fake, fake, fake, fake, fake, null, 1, 128, 128, 0.1,
                                  ctypes.byref(bl), 0, 0, null, null, null) == ops.CALIB_ERR_INVALID
    assert L.sparse_attn_fwd_host(fake, fake, fake, fake, fake, fake, fake, fake, null, 1, 128, 96, 0.1,
                                  ctypes.byref(bl), 0, 1, null, null, null) == ops.CALIB_ERR_UNSUPPORTED
    assert L.sparse_attn_fwd_host(fake, fake, fake, fake, fake, fake, fake, fake, null, 1, 128, 128, 0.1,
                                  ctypes.byref(bl2), 0, 1, null, null, null) == ops.CALIB_ERR_INVALID
    rep = (ctypes.c_uint8 * 1)(1)
    assert L.sparse_attn_fwd_repeat_host(null, fake, fake, fake, fake, fake, fake, fake, null, 1, 128, 1, 1, 128,
                                         0, 1, ctypes.cast(rep, ctypes.c_void_p), 0.1, ctypes.byref(bl), 0, 1,
                                         null, null, null) == ops.CALIB_ERR_INVALID
    assert L.sparse_attn_fwd_repeat_host(fake, fake, fake, fake, fake, fake, fake, fake, null, 1, 128, 1, 1, 128,
                                         0, 1, null, 0.1, ctypes.byref(bl), 0, 1, null, null,
                                         null) == ops.CALIB_ERR_INVALID
    # selection beyond nk = 1024 is unsupported
    assert L.calib_select_mask(fake, 1, 1, 1025, 0.9, null, fake, null, null) in (
        ops.CALIB_ERR_UNSUPPORTED,)
    # energy pass beyond N = 131072 tokens is unsupported
    assert L.calib_block_energy(fake, fake, null, 1, 131073, 128, 128, 0.1, null, 0, fake, 0, null) == \
        ops.CALIB_ERR_UNSUPPORTED


def test_plain_c_client(tmp_path):
    """The header compiles as C99 and a C program linked to the library gets the documented
    answers from the host-decided paths (tests/abi_client.c), with no Python in between."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    ops.lib()                                          # the library exists (built in-tree)
    libdir = os.path.dirname(ops.LIB_PATH)
    exe = str(tmp_path / "abi_client")
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "abi_client.c"), "-L", libdir, "-lcalibatt", f"-Wl,-rpath,{libdir}",
           "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    res = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0 and res.stdout.strip() == "ok", res.stdout + res.stderr


def test_product_path_refuses_host_tensors_and_a_missing_library(monkeypatch):
    """No CPU fallback: device entry points reject CPU tensors before any call, and a
    missing shared library raises instead of degrading to another implementation."""
    import torch
    q = torch.zeros(1, 128, 128, dtype=torch.bfloat16)
    m = torch.ones(1, 1, 1, dtype=torch.uint8)
    bl = ops.BlockList(1, 1, 1, 128, torch.zeros(2, dtype=torch.int32), torch.zeros(1, dtype=torch.int16))
    with pytest.raises(TypeError, match="CUDA tensor"):
        ops.sparse_attn_fwd(q, q, q, bl)
    with pytest.raises(TypeError, match="CUDA tensor"):
        ops.block_energy(q, q, 128)
    with pytest.raises(TypeError, match="CUDA tensor"):
        ops.select_mask(torch.zeros(1, 1, 1), 0.9)
    with pytest.raises(TypeError, match="CUDA tensor"):
        ops.mask_to_csr(m)
    if not torch.cuda.is_available():
        with pytest.raises(Exception):
            ops.sparse_attn_fwd_host(q, q, q, bl)       # needs a device for its staging buffers
    monkeypatch.setattr(ops, "_lib", None)
    monkeypatch.setattr(ops, "LIB_PATH", os.path.join(ROOT, "no_such_dir", "libcalibatt.so"))
    with pytest.raises(RuntimeError, match="missing"):
        ops.lib()
