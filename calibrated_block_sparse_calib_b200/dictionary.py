"""The calibrated mask dictionary: one static block mask per (timestep t, layer l, head h).

The method calibrates offline and keeps, per timestep, layer and head, a static block mask
(plus the spatial-repetition flag of the head) that inference looks up instead of searching
([zh] §2.2A-§2.2B, [de] §2A.5 and §2B, [fr] §2.B.3 and §2.C of the summaries of
"Accelerating Text-to-Video Generation with Calibrated Sparse Attention").  Here one
(t, l) slice covers all H heads:

* on the device, a slice is kept in interval form (runs of consecutive kept key blocks per
  row, calib_csr_to_intervals) and expanded on demand into the CSR skip list plus the
  longest-first schedule the attention kernel walks (calib_intervals_to_csr,
  calib_build_schedule);
* on disk, the dictionary is one little-endian file that also records how it was
  calibrated -- the aggregation over calibration inputs, the vote threshold rho, the number
  of inputs, the repetition threshold gamma, and each slice's selection threshold eps(t),
  which the method varies with the timestep ([fr] §2.B.1, §2.B.2, §2.B.3):

      b"CBSDICT2"
      int32[12] T, L, H, nq, nk, block, stride, n_slices,
                rho_num, rho_den, mode (0 vote, 1 energy mean, 2 masks given as they are),
                n_inputs (0 when not recorded)
      float64   gamma (NaN when no repetition detection ran)
      n_slices x {
          int32[3]  t, l, n_runs
          float64   tau of the slice (0 when not recorded)
          uint8[H]  repeat flag of every head, zero-padded to a multiple of 4 bytes
          int32[H*nq + 1]  run offsets per row
          int16[n_runs]    run starts
          int16[n_runs]    run lengths, zero-padded to a multiple of 4 bytes
      }

Repeat heads use anchor-space query blocks: their rows past the anchor sequence are empty.
Every conversion runs in the library's kernels; this module moves buffers and bytes, and
checks a file's header and run structure on the host before any of it reaches the device:
a file that is truncated, has trailing bytes, or whose runs could not come from a mask (or
would expand to more than 2^31 - 1 kept blocks, the int32 offsets of the skip list) is
refused with ValueError.  Files of the first format (b"CBSDICT1", which recorded no
calibration parameters) are refused with a message saying so.
"""
from __future__ import annotations

import math
import struct
from dataclasses import dataclass, field
from typing import Dict, Optional, Sequence, Tuple

import numpy as np
import torch

from . import ops

MAGIC = b"CBSDICT2"
MAGIC_V1 = b"CBSDICT1"
MODES = ("vote", "energy_mean", "given")
_INT32_MAX = 2**31 - 1


def _check_runs(key, iv_ptr: np.ndarray, starts: np.ndarray, lens: np.ndarray, n: int, nk: int):
    """A slice read from a file must describe a valid skip list before it is expanded on
    the device: offsets from 0 to n, non-decreasing; every run non-empty and inside
    [0, nk); runs of a row ascending and disjoint (each starts past the previous one's end)."""
    ptr = iv_ptr.astype(np.int64)
    if ptr[0] != 0 or ptr[-1] != n or np.any(np.diff(ptr) < 0):
        raise ValueError(f"slice {key}: run offsets must rise from 0 to {n}")
    st, ln = starts.astype(np.int64), lens.astype(np.int64)
    if n and (st.min() < 0 or ln.min() < 1 or (st + ln).max() > nk):
        raise ValueError(f"slice {key}: a run is empty or outside the {nk} key blocks")
    if int(ln.sum()) > _INT32_MAX:
        raise ValueError(f"slice {key}: its runs expand to more than 2^31 - 1 kept blocks")
    row = np.repeat(np.arange(ptr.size - 1), np.diff(ptr))
    same = row[1:] == row[:-1]
    if np.any(st[1:][same] < (st + ln)[:-1][same]):
        raise ValueError(f"slice {key}: runs of a row overlap or are out of order")


@dataclass
class _Slice:
    iv_ptr: torch.Tensor          # int32 [H*nq + 1]
    starts: torch.Tensor          # int16 [n_runs]
    lens: torch.Tensor            # int16 [n_runs]
    repeat: Tuple[bool, ...]      # [H]
    tau: float = 0.0              # selection threshold eps(t) of the slice (0: not recorded)


@dataclass
class MaskDictionary:
    T: int
    L: int
    H: int
    nq: int
    nk: int
    block: int
    stride: int = 1
    rho: Tuple[int, int] = (1, 2)          # vote threshold rho = rho[0] / rho[1]
    mode: str = "vote"                     # "vote", "energy_mean" or "given"
    n_inputs: int = 0                      # calibration inputs (0: not recorded)
    gamma: Optional[float] = None          # repetition threshold (None: no detection ran)
    slices: Dict[Tuple[int, int], _Slice] = field(default_factory=dict)
    _lists: Dict[Tuple[int, int], ops.BlockList] = field(default_factory=dict, repr=False)

    # ---- building ----------------------------------------------------------------
    def put_mask(self, t: int, l: int, mask: torch.Tensor, repeat: Optional[Sequence[bool]] = None,
                 tau: float = 0.0):
        """Store the (t, l) slice from a uint8 [H, nq, nk] device mask (anchor-space rows for
        repeat heads), calibrated at threshold `tau`."""
        self._check_key(t, l)
        if tuple(mask.shape) != (self.H, self.nq, self.nk):
            raise ValueError(f"mask shape {tuple(mask.shape)} != {(self.H, self.nq, self.nk)}")
        row_ptr, col_idx = ops.mask_to_csr(mask)
        self.put_csr(t, l, row_ptr, col_idx, repeat, tau)

    def put_csr(self, t: int, l: int, row_ptr: torch.Tensor, col_idx: torch.Tensor,
                repeat: Optional[Sequence[bool]] = None, tau: float = 0.0):
        self._check_key(t, l)
        iv_ptr, starts, lens = ops.csr_to_intervals(row_ptr, col_idx, self.H, self.nq)
        rep = tuple(bool(x) for x in (repeat if repeat is not None else [False] * self.H))
        if len(rep) != self.H:
            raise ValueError("repeat needs one flag per head")
        if not 0.0 <= float(tau) <= 1.0:
            raise ValueError("tau must be in [0, 1] (0: not recorded)")
        self.slices[(t, l)] = _Slice(iv_ptr, starts.clone(), lens.clone(), rep, float(tau))
        self._lists.pop((t, l), None)

    def tau(self, t: int, l: int) -> float:
        """The selection threshold slice (t, l) was calibrated at (0 when not recorded)."""
        return self.slices[(t, l)].tau

    # ---- lookup ------------------------------------------------------------------
    def block_list(self, t: int, l: int) -> ops.BlockList:
        """CSR skip list + schedule of slice (t, l), expanded on first use and cached."""
        key = (t, l)
        if key not in self._lists:
            s = self.slices[key]
            row_ptr, col_idx = ops.intervals_to_csr(s.iv_ptr, s.starts, s.lens, self.H, self.nq)
            work = ops.build_schedule(row_ptr, self.H, self.nq)
            self._lists[key] = ops.BlockList(self.H, self.nq, self.nk, self.block, row_ptr, col_idx,
                                             work).validate()
        return self._lists[key]

    def repeat_heads(self, t: int, l: int) -> Tuple[bool, ...]:
        return self.slices[(t, l)].repeat

    def _check_key(self, t: int, l: int):
        if not (0 <= t < self.T and 0 <= l < self.L):
            raise KeyError(f"(t, l) = {(t, l)} outside T={self.T}, L={self.L}")

    # ---- files -------------------------------------------------------------------
    def _header_fields(self):
        if self.mode not in MODES:
            raise ValueError(f"mode must be one of {MODES}")
        rn, rd = (int(x) for x in self.rho)
        if not (0 <= rn <= rd and rd >= 1):
            raise ValueError("rho must be a fraction in [0, 1]")
        gamma = math.nan if self.gamma is None else float(self.gamma)
        return rn, rd, MODES.index(self.mode), int(self.n_inputs), gamma

    def to_bytes(self) -> bytes:
        rn, rd, mode, n_in, gamma = self._header_fields()
        out = [MAGIC, struct.pack("<12i", self.T, self.L, self.H, self.nq, self.nk, self.block, self.stride,
                                  len(self.slices), rn, rd, mode, n_in), struct.pack("<d", gamma)]
        for (t, l) in sorted(self.slices):
            s = self.slices[(t, l)]
            n = s.starts.numel()
            out.append(struct.pack("<3id", t, l, n, float(s.tau)))
            rep = np.array(s.repeat, np.uint8).tobytes()
            out.append(rep + b"\0" * (-len(rep) % 4))
            out.append(s.iv_ptr.cpu().numpy().astype("<i4").tobytes())
            runs = s.starts.cpu().numpy().astype("<i2").tobytes() + s.lens.cpu().numpy().astype("<i2").tobytes()
            out.append(runs + b"\0" * (-len(runs) % 4))
        return b"".join(out)

    def save(self, path: str):
        with open(path, "wb") as f:
            f.write(self.to_bytes())

    @classmethod
    def from_bytes(cls, buf: bytes, device="cuda") -> "MaskDictionary":
        if buf[:8] == MAGIC_V1:
            raise ValueError("a CBSDICT1 dictionary records no calibration parameters (tau, rho, mode); "
                             "this version reads CBSDICT2 only -- rebuild the dictionary")
        if buf[:8] != MAGIC:
            raise ValueError("not a calibrated mask dictionary (bad magic)")

        def need(off, size, what):
            if off + size > len(buf):
                raise ValueError(f"file truncated in {what} ({len(buf)} bytes, need {off + size})")

        need(8, 56, "the header")
        T, L, H, nq, nk, block, stride, n_slices, rn, rd, mode, n_in = struct.unpack_from("<12i", buf, 8)
        (gamma,) = struct.unpack_from("<d", buf, 56)
        if min(T, L, H, nq, nk, stride) < 1 or block not in (64, 128) or nk > 32767 or n_slices < 0:
            raise ValueError(f"bad header {(T, L, H, nq, nk, block, stride, n_slices)}")
        if H * nq * nk > _INT32_MAX:
            raise ValueError(f"bad header: H*nq*nk = {H * nq * nk} exceeds 2^31 - 1")
        if not (0 <= rn <= rd and rd >= 1) or not 0 <= mode < len(MODES) or n_in < 0:
            raise ValueError(f"bad calibration record rho={rn}/{rd} mode={mode} n_inputs={n_in}")
        d = cls(T, L, H, nq, nk, block, stride, rho=(rn, rd), mode=MODES[mode], n_inputs=n_in,
                gamma=None if math.isnan(gamma) else gamma)
        off = 64
        for _ in range(n_slices):
            need(off, 20, "a slice record")
            t, l, n, tau = struct.unpack_from("<3id", buf, off)
            off += 20
            key = (t, l)
            if not 0 <= n <= H * nq * nk:
                raise ValueError(f"slice {key}: {n} runs for {H * nq} rows of {nk} blocks")
            if not 0.0 <= tau <= 1.0:
                raise ValueError(f"slice {key}: tau {tau} outside [0, 1]")
            size = H + (-H % 4) + 4 * (H * nq + 1) + 4 * n
            need(off, size, f"slice {key}")
            rep = tuple(bool(x) for x in np.frombuffer(buf, np.uint8, H, off))
            off += H + (-H % 4)
            iv_ptr = np.frombuffer(buf, "<i4", H * nq + 1, off).astype(np.int32)
            off += 4 * (H * nq + 1)
            starts = np.frombuffer(buf, "<i2", n, off).astype(np.int16)
            lens = np.frombuffer(buf, "<i2", n, off + 2 * n).astype(np.int16)
            off += 4 * n
            _check_runs(key, iv_ptr, starts, lens, n, nk)
            d._check_key(t, l)
            d.slices[key] = _Slice(torch.from_numpy(iv_ptr.copy()).to(device),
                                   torch.from_numpy(starts.copy()).to(device),
                                   torch.from_numpy(lens.copy()).to(device), rep, float(tau))
        if off != len(buf):
            raise ValueError(f"{len(buf) - off} trailing bytes")
        return d

    @classmethod
    def load(cls, path: str, device="cuda") -> "MaskDictionary":
        with open(path, "rb") as f:
            return cls.from_bytes(f.read(), device)
