"""Offline calibration of one (timestep, layer) slice: the sequence of library calls the
method prescribes, from calibration inputs to the slice's block masks and repeat flags.

For every head of the slice ([zh] §2.2A, [de] §2A.1-§2A.5, [fr] §2.B of the summaries of
"Accelerating Text-to-Video Generation with Calibrated Sparse Attention"):

1. spatial-repetition detection (optional, gamma given): cosines between sampled tokens'
   attention rows and their anchors' over all inputs (calib_repeat_similarity), and the
   per-head decision mean > gamma (calib_repeat_flags);
2. block energies per input, over all query rows (calib_block_energy), and over the anchor
   rows for the flagged heads (their masks live in anchor query-block space);
3. either the pages' vote -- per-input minimal tau-selection of all inputs in one batched
   launch that accumulates the vote counts (calib_select_mask_batched), then the
   cross-input vote (calib_aggregate_masks) -- or the energy mean: energies summed over the
   inputs (the energy kernel's accumulate flag), divided by the number of inputs
   (calib_energy_mean) and selected once (calib_select_mask);
4. the slice mask: a flagged head takes its anchor-space rows (the rest of its rows stay
   empty), the others their full-space rows.

tau may differ per timestep (the pages keep early timesteps stricter); the caller passes
the slice's value.  Every arithmetic step runs in the library's kernels; this module
sequences calls and moves buffers.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch

from . import ops


def calibrate_slice(inputs: List[Tuple[torch.Tensor, torch.Tensor]], F: int, Hl: int, Wl: int, n_text: int,
                    block: int, tau: float, rho: Sequence[int] = (1, 2), mode: str = "vote",
                    gamma: Optional[float] = None, stride: int = 4, members: Optional[torch.Tensor] = None,
                    force_keep: Optional[torch.Tensor] = None, force_keep_anchor: Optional[torch.Tensor] = None):
    """Returns (mask uint8 [H, nq, nk], repeat bool list [H], details dict).

    inputs     : per calibration input, (q, k) bf16 [H, N, D] on the device.
    mode       : "vote" (per-input masks, strict vote above rho) or "energy_mean" (block
                 energies averaged over the inputs, then one selection).
    gamma      : repetition threshold, or None to skip detection (no head repeats).
    members    : int32 [n] sampled video tokens for detection (required with gamma).
    force_keep : uint8 [H, nq, nk] blocks always kept (e.g. text rows / columns).
    force_keep_anchor : the same in anchor query-block space [H, nq_anchor, nk]; required
                 with force_keep when a head is flagged (text rows sit at the end of the
                 compacted anchor sequence, so the full-space rows do not carry over).
    """
    if mode not in ("vote", "energy_mean"):
        raise ValueError("mode must be 'vote' or 'energy_mean'")
    q0, k0 = inputs[0]
    H, N, D = q0.shape
    dev = q0.device
    nq = nk = ops.nblocks(N, block)

    # 1. repetition detection
    repeat = [False] * H
    details = {}
    if gamma is not None:
        if members is None:
            raise ValueError("repetition detection needs sampled tokens (members)")
        cos = torch.cat([ops.repeat_similarity(q, k, members, F, Hl, Wl, stride, block) for q, k in inputs], dim=1)
        mem_all = members.repeat(len(inputs))
        mean, flag = ops.repeat_flags(cos, mem_all, F, Hl, Wl, stride, gamma)
        repeat = [bool(x) for x in flag.cpu().tolist()]
        details["repeat_mean"] = mean.cpu().tolist()

    # 2-3. energies and selection, full space and (if needed) anchor space
    def select_space(q_rows=None, nq_space=nq, force=None):
        shape = (H, nq_space, nk)
        n_in = len(inputs)
        if mode == "vote":
            energies = torch.empty((n_in,) + shape, dtype=torch.float32, device=dev)
            for d, (q, k) in enumerate(inputs):
                ops.block_energy(q, k, block, q_rows=q_rows, out=energies[d])
            counts = torch.zeros(shape, dtype=torch.int32, device=dev)
            ops.select_mask_batched(energies, [tau] * n_in, force_keep=force, count_accum=counts,
                                    write_masks=False)
            return ops.aggregate_masks(counts, n_in, rho)
        esum = None
        for d, (q, k) in enumerate(inputs):
            esum = ops.block_energy(q, k, block, q_rows=q_rows, out=esum, accumulate=d > 0)
        return ops.select_mask(ops.energy_mean(esum, n_in, out=esum), tau, force_keep=force)

    mask = select_space(force=force_keep)
    if any(repeat):
        rows = ops.anchor_rows(F, Hl, Wl, n_text, stride, device=dev)
        nq_a = ops.nblocks(rows.numel(), block)
        if force_keep is not None and force_keep_anchor is None:
            raise ValueError("force_keep needs force_keep_anchor once a head is flagged")
        mask_a = select_space(q_rows=rows, nq_space=nq_a, force=force_keep_anchor)
        for h in range(H):
            if repeat[h]:
                mask[h].zero_()
                mask[h, :nq_a].copy_(mask_a[h])
        details["nq_anchor"] = nq_a
    return mask, repeat, details
