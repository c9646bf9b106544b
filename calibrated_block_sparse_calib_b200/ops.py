"""ctypes binding of libcalibatt.so (see include/calibatt.h for the semantics).

Argument marshalling only: every function checks dtypes, shapes and devices, allocates
outputs with torch (device memory), and calls the C ABI on torch's current CUDA stream.
All arithmetic runs in the library's sm_100a kernels.  There is no fallback: a missing
library or a non-CUDA tensor raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcalibatt.so")

CALIB_OK, CALIB_ERR_INVALID, CALIB_ERR_UNSUPPORTED, CALIB_ERR_CUDA, CALIB_ERR_TIMEOUT = range(5)
CALIB_ATTN_OUT_F32 = 1


class CalibError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")


class _BlockListC(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("nq", ctypes.c_int32), ("nk", ctypes.c_int32),
                ("block", ctypes.c_int32), ("row_ptr", ctypes.c_void_p), ("col_idx", ctypes.c_void_p),
                ("work", ctypes.c_void_p), ("n_work", ctypes.c_int32)]


_lib = None
_P, _I, _F, _D, _U32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_double, ctypes.c_uint32
_SIGS = {
    "calib_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "calib_device_check": ([_P], ctypes.c_int),
    "calib_block_energy": ([_P, _P, _P, _I, _I, _I, _I, _F, _P, _I, _P, _I, _P], ctypes.c_int),
    "calib_select_mask": ([_P, _I, _I, _I, _D, _P, _P, _P, _P], ctypes.c_int),
    "calib_select_mask_batched": ([_P, _I, _I, _I, _I, _P, _P, _P, _P, _P], ctypes.c_int),
    "calib_energy_mean": ([_P, ctypes.c_int64, _I, _P, _P], ctypes.c_int),
    "calib_validate_block_list_host": ([_I, _I, _I, _P, _P, ctypes.c_int64, _P, _I], ctypes.c_int),
    "calib_aggregate_masks": ([_P, _I, _I, _I, _I, _I, _I, _P, _P], ctypes.c_int),
    "calib_mask_to_csr": ([_P, _I, _I, _I, _P, _P, _P], ctypes.c_int),
    "calib_build_schedule": ([_P, _I, _I, _P, _P], ctypes.c_int),
    "calib_csr_to_intervals": ([_P, _P, _I, _I, _P, _P, _P, _P], ctypes.c_int),
    "calib_repeat_similarity": ([_P, _P, _P, _I, _I, _I, _I, _F, _I, _I, _I, _I, _P, _I, _P, _P], ctypes.c_int),
    "calib_repeat_flags": ([_P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P], ctypes.c_int),
    "calib_intervals_to_csr": ([_P, _P, _P, _I, _I, _P, _P, _P], ctypes.c_int),
    "calib_anchor_count": ([_I, _I, _I, _I, _I], ctypes.c_int64),
    "calib_anchor_rows": ([_I, _I, _I, _I, _I, _P, _P], ctypes.c_int),
    "sparse_attn_fwd": ([_P, _P, _P, _P, _P, _I, _I, _I, _F, ctypes.POINTER(_BlockListC), _U32, _P],
                        ctypes.c_int),
    "sparse_attn_fwd_repeat": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _F,
                                ctypes.POINTER(_BlockListC), _U32, _P], ctypes.c_int),
    "sparse_attn_fwd_host": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _F, ctypes.POINTER(_BlockListC),
                              _U32, _I, _P, _P, _P], ctypes.c_int),
    "sparse_attn_fwd_repeat_host": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _F,
                                     ctypes.POINTER(_BlockListC), _U32, _I, _P, _P, _P], ctypes.c_int),
    "calib_selftest_wait_timeout": ([_U32, _P], ctypes.c_int),
}


def lib():
    """Load libcalibatt.so (built in-tree); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m calibrated_block_sparse_calib_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().calib_status_string(int(s)).decode()


def _check(fn: str, s: int):
    if s != CALIB_OK:
        raise CalibError(fn, s)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def device_check():
    """Synchronise the current stream and raise if a kernel recorded an error."""
    _check("calib_device_check", lib().calib_device_check(_stream()))


def selftest_wait_timeout(timeout_us: int = 1000) -> int:
    """Run the bounded-wait self-test; returns the status (CALIB_ERR_TIMEOUT expected)."""
    return lib().calib_selftest_wait_timeout(int(timeout_us), _stream())


def nblocks(n: int, block: int) -> int:
    return (n + block - 1) // block


# ----------------------------------------------------------------------------------
# calibration
# ----------------------------------------------------------------------------------

def block_energy(q: torch.Tensor, k: torch.Tensor, block: int, scale: Optional[float] = None,
                 lse: Optional[torch.Tensor] = None, q_rows: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None, accumulate: bool = False) -> torch.Tensor:
    """fp32 block energies [H, ceil(Nq/B), ceil(N/B)] of softmax(scale q k^T)."""
    H, N, D = k.shape
    _need(q, "q", torch.bfloat16, (H, N, D))
    _need(k, "k", torch.bfloat16)
    Nq = N
    if q_rows is not None:
        _need(q_rows, "q_rows", torch.int32)
        Nq = q_rows.numel()
    if lse is not None:
        _need(lse, "lse", torch.float32, (H, Nq))
    shape = (H, nblocks(Nq, block), nblocks(N, block))
    if out is None:
        out = (torch.zeros if accumulate else torch.empty)(shape, dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, shape)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    _check("calib_block_energy", lib().calib_block_energy(
        _ptr(q), _ptr(k), _ptr(lse), H, N, D, block, scale, _ptr(q_rows), Nq if q_rows is not None else 0,
        _ptr(out), 1 if accumulate else 0, _stream()))
    return out


def select_mask(energy: torch.Tensor, tau: float, force_keep: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None, count_accum: Optional[torch.Tensor] = None) -> torch.Tensor:
    """uint8 keep mask [H, nq, nk] of the minimal tau-energy selection."""
    _need(energy, "energy", torch.float32)
    H, nq, nk = energy.shape
    if force_keep is not None:
        _need(force_keep, "force_keep", torch.uint8, energy.shape)
    if out is None:
        out = torch.empty(energy.shape, dtype=torch.uint8, device=energy.device)
    _need(out, "out", torch.uint8, energy.shape)
    if count_accum is not None:
        _need(count_accum, "count_accum", torch.int32, energy.shape)
    _check("calib_select_mask", lib().calib_select_mask(
        _ptr(energy), H, nq, nk, float(tau), _ptr(force_keep), _ptr(out), _ptr(count_accum), _stream()))
    return out


def select_mask_batched(energy: torch.Tensor, taus: Sequence[float], force_keep: Optional[torch.Tensor] = None,
                        out: Optional[torch.Tensor] = None, count_accum: Optional[torch.Tensor] = None,
                        write_masks: bool = True) -> Optional[torch.Tensor]:
    """Minimal tau-energy selection of a batch energy[b] (fp32 [nb, H, nq, nk]) at taus[b], in
    one launch.  Returns the uint8 masks [nb, H, nq, nk] (None with write_masks=False, when
    only count_accum [H, nq, nk] is wanted: it is incremented by the number of entries that
    keep each block)."""
    _need(energy, "energy", torch.float32)
    nb, H, nq, nk = energy.shape
    taus = [float(t) for t in taus]
    if len(taus) != nb:
        raise ValueError(f"need one tau per batch entry ({nb}), got {len(taus)}")
    if force_keep is not None:
        _need(force_keep, "force_keep", torch.uint8, (H, nq, nk))
    if count_accum is not None:
        _need(count_accum, "count_accum", torch.int32, (H, nq, nk))
    if write_masks:
        if out is None:
            out = torch.empty(energy.shape, dtype=torch.uint8, device=energy.device)
        _need(out, "out", torch.uint8, energy.shape)
    else:
        out = None
        if count_accum is None:
            raise ValueError("write_masks=False needs count_accum")
    tau_arr = (ctypes.c_double * nb)(*taus)
    _check("calib_select_mask_batched", lib().calib_select_mask_batched(
        _ptr(energy), nb, H, nq, nk, ctypes.cast(tau_arr, ctypes.c_void_p), _ptr(force_keep), _ptr(out),
        _ptr(count_accum), _stream()))
    return out


def energy_mean(energy_sum: torch.Tensor, n_inputs: int, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """fp32 energies averaged over n_inputs calibration inputs (energy_sum / n_inputs); `out`
    may be energy_sum itself."""
    _need(energy_sum, "energy_sum", torch.float32)
    if out is None:
        out = torch.empty_like(energy_sum)
    _need(out, "out", torch.float32, energy_sum.shape)
    _check("calib_energy_mean", lib().calib_energy_mean(
        _ptr(energy_sum), energy_sum.numel(), int(n_inputs), _ptr(out), _stream()))
    return out


def validate_block_list_host(H: int, nq: int, nk: int, row_ptr, col_idx, work=None) -> bool:
    """True when a skip list held in host memory (numpy arrays or CPU tensors) is well formed
    for the attention calls (calib_validate_block_list_host); no device work."""
    import numpy as np
    rp = np.ascontiguousarray(np.asarray(row_ptr), dtype=np.int32)
    ci = np.ascontiguousarray(np.asarray(col_idx), dtype=np.int16)
    if rp.shape != (H * nq + 1,):
        return False
    wk = None if work is None else np.ascontiguousarray(np.asarray(work), dtype=np.int32)
    s = lib().calib_validate_block_list_host(
        int(H), int(nq), int(nk), rp.ctypes.data_as(ctypes.c_void_p),
        ci.ctypes.data_as(ctypes.c_void_p) if ci.size else None, int(ci.size),
        None if wk is None else wk.ctypes.data_as(ctypes.c_void_p), 0 if wk is None else int(wk.size))
    return s == CALIB_OK


def aggregate_masks(counts: torch.Tensor, n_inputs: int, rho: Sequence[int] = (1, 2),
                    out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """uint8 mask of blocks kept with frequency strictly above rho = rho[0]/rho[1]."""
    _need(counts, "counts", torch.int32)
    H, nq, nk = counts.shape
    if out is None:
        out = torch.empty(counts.shape, dtype=torch.uint8, device=counts.device)
    _need(out, "out", torch.uint8, counts.shape)
    _check("calib_aggregate_masks", lib().calib_aggregate_masks(
        _ptr(counts), H, nq, nk, int(n_inputs), int(rho[0]), int(rho[1]), _ptr(out), _stream()))
    return out


def mask_to_csr(mask: torch.Tensor):
    """(row_ptr int32 [H*nq+1], col_idx int16 [H*nq*nk] capacity) skip list of a mask."""
    _need(mask, "mask", torch.uint8)
    H, nq, nk = mask.shape
    row_ptr = torch.empty(H * nq + 1, dtype=torch.int32, device=mask.device)
    col_idx = torch.empty(max(1, H * nq * nk), dtype=torch.int16, device=mask.device)
    _check("calib_mask_to_csr", lib().calib_mask_to_csr(
        _ptr(mask), H, nq, nk, _ptr(row_ptr), _ptr(col_idx), _stream()))
    return row_ptr, col_idx


def csr_to_intervals(row_ptr: torch.Tensor, col_idx: torch.Tensor, H: int, nq: int):
    """Runs of consecutive kept blocks per row: (iv_ptr int32 [H*nq+1], starts int16, lengths
    int16), the runs trimmed to their count."""
    _need(row_ptr, "row_ptr", torch.int32, (H * nq + 1,))
    _need(col_idx, "col_idx", torch.int16)
    cap = max(1, col_idx.numel())
    iv_ptr = torch.empty(H * nq + 1, dtype=torch.int32, device=row_ptr.device)
    starts = torch.empty(cap, dtype=torch.int16, device=row_ptr.device)
    lens = torch.empty(cap, dtype=torch.int16, device=row_ptr.device)
    _check("calib_csr_to_intervals", lib().calib_csr_to_intervals(
        _ptr(row_ptr), _ptr(col_idx), H, nq, _ptr(iv_ptr), _ptr(starts), _ptr(lens), _stream()))
    n = int(iv_ptr[-1].item())
    return iv_ptr, starts[:n], lens[:n]


def intervals_to_csr(iv_ptr: torch.Tensor, starts: torch.Tensor, lens: torch.Tensor, H: int, nq: int):
    """CSR skip list (row_ptr int32 [H*nq+1], col_idx int16 [nnz]) from runs: one call
    sizes the list (row_ptr only), the second fills it."""
    _need(iv_ptr, "iv_ptr", torch.int32, (H * nq + 1,))
    _need(starts, "starts", torch.int16)
    _need(lens, "lens", torch.int16, starts.shape)
    dev = iv_ptr.device
    # an empty run list still needs valid pointers
    st = starts if starts.numel() else torch.zeros(1, dtype=torch.int16, device=dev)
    ln = lens if lens.numel() else torch.zeros(1, dtype=torch.int16, device=dev)
    row_ptr = torch.empty(H * nq + 1, dtype=torch.int32, device=dev)
    _check("calib_intervals_to_csr", lib().calib_intervals_to_csr(
        _ptr(iv_ptr), _ptr(st), _ptr(ln), H, nq, _ptr(row_ptr), None, _stream()))
    nnz = int(row_ptr[-1].item())
    col_idx = torch.empty(max(1, nnz), dtype=torch.int16, device=dev)
    _check("calib_intervals_to_csr", lib().calib_intervals_to_csr(
        _ptr(iv_ptr), _ptr(st), _ptr(ln), H, nq, _ptr(row_ptr), _ptr(col_idx), _stream()))
    return row_ptr, col_idx[:nnz]


def repeat_similarity(q: torch.Tensor, k: torch.Tensor, members: torch.Tensor, F: int, Hl: int, Wl: int,
                      stride: int, block: int = 128, scale: Optional[float] = None,
                      lse: Optional[torch.Tensor] = None) -> torch.Tensor:
    """fp32 [H, n]: cosine between the attention rows of each sampled token and its anchor."""
    H, N, D = k.shape
    _need(q, "q", torch.bfloat16, (H, N, D))
    _need(k, "k", torch.bfloat16)
    _need(members, "members", torch.int32)
    if lse is not None:
        _need(lse, "lse", torch.float32, (H, N))
    n = members.numel()
    out = torch.empty((H, n), dtype=torch.float32, device=q.device)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    _check("calib_repeat_similarity", lib().calib_repeat_similarity(
        _ptr(q), _ptr(k), _ptr(lse), H, N, D, block, scale, F, Hl, Wl, stride, _ptr(members), n, _ptr(out),
        _stream()))
    return out


def repeat_flags(cos: torch.Tensor, members: torch.Tensor, F: int, Hl: int, Wl: int, stride: int, gamma: float):
    """(mean fp32 [H], flag uint8 [H]): mean similarity over non-anchor samples, flag mean > gamma."""
    _need(cos, "cos", torch.float32)
    _need(members, "members", torch.int32)
    H, n = cos.shape
    mean = torch.empty(H, dtype=torch.float32, device=cos.device)
    flag = torch.empty(H, dtype=torch.uint8, device=cos.device)
    _check("calib_repeat_flags", lib().calib_repeat_flags(
        _ptr(cos), _ptr(members), H, n, F, Hl, Wl, stride, float(gamma), _ptr(mean), _ptr(flag), _stream()))
    return mean, flag


def build_schedule(row_ptr: torch.Tensor, H: int, nq: int) -> torch.Tensor:
    """int32 work list (h << 16 | i): heads in order, longest rows first within a head."""
    _need(row_ptr, "row_ptr", torch.int32, (H * nq + 1,))
    work = torch.empty(H * nq, dtype=torch.int32, device=row_ptr.device)
    _check("calib_build_schedule", lib().calib_build_schedule(_ptr(row_ptr), H, nq, _ptr(work), _stream()))
    return work


def anchor_count(F: int, Hl: int, Wl: int, n_text: int, stride: int) -> int:
    n = lib().calib_anchor_count(F, Hl, Wl, n_text, stride)
    if n < 0:
        raise ValueError("invalid anchor geometry")
    return int(n)


def anchor_rows(F: int, Hl: int, Wl: int, n_text: int, stride: int, device="cuda") -> torch.Tensor:
    """int32 token indices of the anchor rows (compacted order)."""
    rows = torch.empty(anchor_count(F, Hl, Wl, n_text, stride), dtype=torch.int32, device=device)
    _check("calib_anchor_rows", lib().calib_anchor_rows(F, Hl, Wl, n_text, stride, _ptr(rows), _stream()))
    return rows


# ----------------------------------------------------------------------------------
# inference
# ----------------------------------------------------------------------------------

@dataclass
class BlockList:
    """Device-resident skip list of one (timestep, layer) slice (see calib_block_list)."""
    H: int
    nq: int
    nk: int
    block: int
    row_ptr: torch.Tensor
    col_idx: torch.Tensor
    work: Optional[torch.Tensor] = None

    def c_struct(self) -> _BlockListC:
        _need(self.row_ptr, "row_ptr", torch.int32, (self.H * self.nq + 1,))
        _need(self.col_idx, "col_idx", torch.int16)
        if self.work is not None:
            _need(self.work, "work", torch.int32)
        return _BlockListC(self.H, self.nq, self.nk, self.block, self.row_ptr.data_ptr(),
                           self.col_idx.data_ptr(), 0 if self.work is None else self.work.data_ptr(),
                           0 if self.work is None else self.work.numel())

    def validate(self) -> "BlockList":
        """Copy the list back to the host and check its structure (rows within col_idx,
        ascending in-range indices, work items in range); raises ValueError if malformed."""
        H, nq, nk = self.H, self.nq, self.nk
        wk = None if self.work is None else self.work.cpu().numpy()
        if not validate_block_list_host(H, nq, nk, self.row_ptr.cpu().numpy(), self.col_idx.cpu().numpy(), wk):
            raise ValueError("malformed skip list")
        return self

    @staticmethod
    def from_mask(mask: torch.Tensor, block: int, schedule: bool = True) -> "BlockList":
        """Skip list (and longest-first schedule) of a uint8 [H, nq, nk] device mask."""
        H, nq, nk = mask.shape
        rp, ci = mask_to_csr(mask)
        work = build_schedule(rp, H, nq) if schedule else None
        return BlockList(H, nq, nk, block, rp, ci, work)


def _out(q, out, out_dtype):
    H, N, D = q.shape
    if out is None:
        out = torch.empty((H, N, D), dtype=out_dtype, device=q.device)
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out must be bf16 or fp32")
    _need(out, "out", out.dtype, (H, N, D))
    return out, (CALIB_ATTN_OUT_F32 if out.dtype == torch.float32 else 0)


def sparse_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, blist: BlockList,
                    scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                    lse: Optional[torch.Tensor] = None, return_lse: bool = False,
                    out_dtype: torch.dtype = torch.bfloat16):
    """Block-sparse attention: O [H, N, D] in bf16 (or fp32 via out_dtype / an fp32 `out`),
    and the fp32 LSE [H, N] if requested."""
    H, N, D = q.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16, (H, N, D))
    out, flags = _out(q, out, out_dtype)
    if return_lse and lse is None:
        lse = torch.empty(H, N, dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, (H, N))
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    cs = blist.c_struct()
    _check("sparse_attn_fwd", lib().sparse_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), H, N, D, scale, ctypes.byref(cs), flags, _stream()))
    return (out, lse) if (return_lse or lse is not None) else out


def sparse_attn_fwd_repeat(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, blist: BlockList,
                           head_repeat: Sequence[bool], F: int, Hl: int, Wl: int, n_text: int, stride: int,
                           scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                           lse: Optional[torch.Tensor] = None, return_lse: bool = False,
                           out_dtype: torch.dtype = torch.bfloat16):
    """Block-sparse attention with spatial repetition on the flagged heads."""
    H, N, D = q.shape
    if N != F * Hl * Wl + n_text:
        raise ValueError("N must equal F*Hl*Wl + n_text")
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16, (H, N, D))
    out, oflags = _out(q, out, out_dtype)
    if return_lse and lse is None:
        lse = torch.empty(H, N, dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, (H, N))
    flags = (ctypes.c_uint8 * H)(*[1 if bool(x) else 0 for x in head_repeat])
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    cs = blist.c_struct()
    _check("sparse_attn_fwd_repeat", lib().sparse_attn_fwd_repeat(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), H, D, F, Hl, Wl, n_text, stride,
        ctypes.cast(flags, ctypes.c_void_p), scale, ctypes.byref(cs), oflags, _stream()))
    return (out, lse) if (return_lse or lse is not None) else out


# ----------------------------------------------------------------------------------
# inference on host tensors: transfers overlapped with the attention, chunk by chunk
# ----------------------------------------------------------------------------------

_copy_streams = {}


def _side_streams(device: torch.device):
    """Two copy streams per device (host -> device and device -> host), created once."""
    key = device.index if device.index is not None else torch.cuda.current_device()
    if key not in _copy_streams:
        with torch.cuda.device(key):
            _copy_streams[key] = (torch.cuda.Stream(), torch.cuda.Stream())
    return _copy_streams[key]


@dataclass
class HostStaging:
    """Device staging buffers for sparse_attn_fwd_host: q, k, v bf16 and o [H, N, D]."""
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    o: torch.Tensor

    @staticmethod
    def allocate(H: int, N: int, D: int, device="cuda", out_dtype: torch.dtype = torch.bfloat16) -> "HostStaging":
        mk = lambda dt: torch.empty((H, N, D), dtype=dt, device=device)
        return HostStaging(mk(torch.bfloat16), mk(torch.bfloat16), mk(torch.bfloat16), mk(out_dtype))


def sparse_attn_fwd_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, blist: BlockList,
                         staging: Optional[HostStaging] = None, out: Optional[torch.Tensor] = None,
                         heads_per_chunk: int = 1, scale: Optional[float] = None,
                         lse: Optional[torch.Tensor] = None, out_dtype: torch.dtype = torch.bfloat16,
                         device=None, repeat: Optional[tuple] = None) -> torch.Tensor:
    """Block-sparse attention of CPU tensors q, k, v (bf16 [H, N, D], pinned for overlap),
    returning O in a CPU tensor (pinned when allocated here).  The call returns once the
    work is queued on the current stream; synchronise it before reading O.
    repeat = (head_repeat, F, Hl, Wl, n_text, stride) selects spatial-repetition mode."""
    H, N, D = q.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if t.device.type != "cpu":
            raise ValueError(f"{n} must be a host tensor")
        if t.dtype != torch.bfloat16 or tuple(t.shape) != (H, N, D) or not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous bf16 [H, N, D]")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if staging is None:
        staging = HostStaging.allocate(H, N, D, dev, out_dtype)
    out_dtype = staging.o.dtype
    for t, n in ((staging.q, "staging.q"), (staging.k, "staging.k"), (staging.v, "staging.v")):
        _need(t, n, torch.bfloat16, (H, N, D))
    _need(staging.o, "staging.o", out_dtype, (H, N, D))
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out must be bf16 or fp32")
    if out is None:
        out = torch.empty((H, N, D), dtype=out_dtype, pin_memory=True)
    if out.device.type != "cpu" or out.dtype != out_dtype or tuple(out.shape) != (H, N, D) or not out.is_contiguous():
        raise ValueError("out must be a contiguous host tensor of the output dtype and shape")
    if lse is not None:
        _need(lse, "lse", torch.float32, (H, N))
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    if staging.q.device.index != torch.cuda.current_device():
        raise ValueError("the staging buffers must be on the current CUDA device")
    h2d, d2h = _side_streams(staging.q.device)
    cs = blist.c_struct()
    flags = CALIB_ATTN_OUT_F32 if out_dtype == torch.float32 else 0
    if repeat is None:
        _check("sparse_attn_fwd_host", lib().sparse_attn_fwd_host(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _ptr(staging.q), _ptr(staging.k),
            _ptr(staging.v), _ptr(staging.o), _ptr(lse), H, N, D, scale, ctypes.byref(cs), flags,
            int(heads_per_chunk), _stream(), h2d.cuda_stream, d2h.cuda_stream))
        return out
    head_repeat, F, Hl, Wl, n_text, stride = repeat
    if N != F * Hl * Wl + n_text:
        raise ValueError("N must equal F*Hl*Wl + n_text")
    rflags = (ctypes.c_uint8 * H)(*[1 if bool(x) else 0 for x in head_repeat])
    _check("sparse_attn_fwd_repeat_host", lib().sparse_attn_fwd_repeat_host(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _ptr(staging.q), _ptr(staging.k),
        _ptr(staging.v), _ptr(staging.o), _ptr(lse), H, D, F, Hl, Wl, n_text, stride,
        ctypes.cast(rflags, ctypes.c_void_p), scale, ctypes.byref(cs), flags, int(heads_per_chunk), _stream(),
        h2d.cuda_stream, d2h.cuda_stream))
    return out

