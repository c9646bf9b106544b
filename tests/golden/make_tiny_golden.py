"""Writes tiny_calibration.json: the float64 oracle's results for the Tiny workload.

    python tests/golden/make_tiny_golden.py

The Tiny workload is 2 heads, head_dim 64, 4 frames of 8 x 16 latent tokens (N = 512),
block 64, three seeded calibration inputs, tau = 0.95, vote above rho = 1/2, and head 1
spatially repetitive at anchor stride 2.  The script calls only the oracle package and
the seeded input generator (which holds none of the method's arithmetic), so every value
in the file comes from the oracle:

  * per input, the block energies in the full query space and in head 1's anchor space
    (oracle.block_energy), stored as the float32 bit patterns that selection reads;
  * per input and space, the tau-selected masks (oracle.select_mask) and their vote
    (oracle.aggregate_masks), in each space;
  * the slice mask (head 0 full space, head 1 anchor space), its skip list
    (oracle.mask_to_csr) and work order (oracle.build_schedule);
  * sampled output rows of the slice's attention on input 0
    (oracle.sparse_attention_repeat), float64.

Rerun it only when a change to the oracle's arithmetic, justified by the pages, changes
these values; tests/test_golden.py checks that the oracle still reproduces the file.
"""
from __future__ import annotations

import hashlib
import json
import math
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from calibrated_block_sparse_calib_b200 import synth  # noqa: E402

OUT = os.path.join(HERE, "tiny_calibration.json")
SAMPLE_ROWS = (0, 16, 37, 53, 63, 64, 130, 146, 255, 256, 300, 383, 400, 511)


def _f64(t):
    import torch
    return t.detach().to("cpu", torch.float32).numpy().astype(np.float64)


def input_digest(q, k, v) -> str:
    """sha256 over the raw bf16 bytes of q, k, v (guards the seeded generator)."""
    import torch
    h = hashlib.sha256()
    for t in (q, k, v):
        h.update(t.contiguous().view(torch.int16).numpy().tobytes())
    return h.hexdigest()


def bits(mask: np.ndarray) -> str:
    return "".join(str(int(x)) for x in np.asarray(mask).reshape(-1))


def f32_words(e: np.ndarray) -> list:
    return [int(w) for w in np.asarray(e, np.float32).reshape(-1).view(np.uint32)]


def compute():
    wl = synth.WORKLOADS["tiny"]
    s = wl.shape
    H, N, D, B = s.H, s.N, s.D, s.block
    tau = float(wl.extra["tau"])
    rho = tuple(int(x) for x in wl.extra["rho"])
    n_in = int(wl.extra["n_calib"])
    stride = int(wl.repeat_stride)
    rep = [h in wl.repeat_heads for h in range(H)]
    scale = 1.0 / math.sqrt(D)
    nb = -(-N // B)
    A = oracle.anchor_rows(s.F, s.Hl, s.Wl, s.n_text, stride)
    nqa = -(-len(A) // B)

    inputs = [synth.make_qkv(wl, input_idx=d) for d in range(n_in)]
    digests = [input_digest(*x) for x in inputs]

    spaces = {"full": None, "anchor": A}
    res = {}
    for name, rows in spaces.items():
        e32s, masks = [], []
        counts = None
        for q, k, _ in inputs:
            e = oracle.block_energy(_f64(q), _f64(k), scale, B, q_rows=rows)
            e32 = e.astype(np.float32)
            m = oracle.select_mask(e32, tau)
            counts = m.astype(np.int64) if counts is None else counts + m
            e32s.append(e32)
            masks.append(m)
        agg = oracle.aggregate_masks(counts, n_in, *rho)
        res[name] = dict(e32=e32s, masks=masks, counts=counts, agg=agg)

    slice_mask = np.zeros((H, nb, nb), np.uint8)
    for h in range(H):
        if rep[h]:
            slice_mask[h, :nqa] = res["anchor"]["agg"][h]
        else:
            slice_mask[h] = res["full"]["agg"][h]
    row_ptr, col_idx = oracle.mask_to_csr(slice_mask)
    work = oracle.build_schedule(row_ptr, H, nb)

    q, k, v = inputs[0]
    O, L = oracle.sparse_attention_repeat(_f64(q), _f64(k), _f64(v), scale, B, slice_mask, rep,
                                          s.F, s.Hl, s.Wl, s.n_text, stride)
    rows = list(SAMPLE_ROWS)
    doc = {
        "about": "Oracle results for the Tiny workload; written by make_tiny_golden.py (oracle only).",
        "sources": {
            "energy": "[zh] 2.2A, [de] 2A.1, [fr] 2.B.1: block energy = sum of post-softmax P over a block",
            "select": "[fr] 2.B.1: fewest key blocks whose cumulative energy reaches tau",
            "vote": "[fr] 2.B.2: keep a block whose keep frequency over the inputs is above rho",
            "skip_list": "[zh] 2.2B, [fr] 2.C: per query block, the kept key blocks",
            "repetition": "[zh] 2.1 / 2.2B, [fr] 2.C: anchor rows computed, broadcast to their group",
            "attention": "[zh] 2.2B, [fr] 2.C: softmax over the kept key blocks only",
        },
        "workload": {"H": H, "N": N, "D": D, "block": B, "F": s.F, "Hl": s.Hl, "Wl": s.Wl,
                     "n_text": s.n_text, "stride": stride, "repeat": rep, "tau": tau,
                     "rho": list(rho), "n_inputs": n_in, "nq": nb, "nq_anchor": nqa,
                     "n_anchor": int(len(A))},
        "inputs_sha256": digests,
        "spaces": {
            name: {
                "shape": list(r["e32"][0].shape),
                "energy_f32_bits": [f32_words(e) for e in r["e32"]],
                "masks": [bits(m) for m in r["masks"]],
                "counts": [int(c) for c in r["counts"].reshape(-1)],
                "vote": bits(r["agg"]),
            }
            for name, r in res.items()
        },
        "slice": {
            "mask": bits(slice_mask),
            "row_ptr": [int(x) for x in row_ptr],
            "col_idx": [int(x) for x in col_idx],
            "work": [int(x) for x in work],
        },
        "attention": {
            "input": 0,
            "rows": rows,
            "O": [[[float(x) for x in O[h, r]] for r in rows] for h in range(H)],
            "LSE": [[float(L[h, r]) for r in rows] for h in range(H)],
        },
    }
    return doc


def main():
    doc = compute()
    with open(OUT, "w") as f:
        json.dump(doc, f, indent=None, separators=(",", ":"))
        f.write("\n")
    print("wrote", OUT, os.path.getsize(OUT), "bytes")


if __name__ == "__main__":
    main()
