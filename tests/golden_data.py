"""Loaders for the fixtures under tests/golden/ (shared by the CPU and GPU tests).

hand_worked.txt holds hand-derived cases (one per line, format in the file's header);
tiny_calibration.json holds the oracle's results for the Tiny workload, written by
tests/golden/make_tiny_golden.py.
"""
from __future__ import annotations

import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _ints(s: str):
    return [int(x) for x in s.split(",") if x != ""]


def _digits(s: str):
    return np.array([int(c) for c in s], np.uint8)


def hand_worked():
    """{"select": [...], "vote": [...], "runs": [...], "anchors": [...]} of parsed cases."""
    cases = {"select": [], "vote": [], "runs": [], "anchors": []}
    with open(os.path.join(GOLDEN, "hand_worked.txt")) as f:
        for ln, line in enumerate(f, 1):
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            kind, *fields = line.split()
            kv = dict(x.split("=", 1) for x in fields)
            c = {"line": ln}
            if kind == "select":
                c["e"] = np.array([float.fromhex(x) if "0x" in x else float(x) for x in kv["e"].split(",")],
                                  np.float32)
                c["tau"] = float.fromhex(kv["tau"]) if "0x" in kv["tau"] else float(kv["tau"])
                c["diag"] = int(kv["diag"])
                c["forced"] = _digits(kv["forced"]).astype(bool) if "forced" in kv else None
                c["keep"] = _digits(kv["keep"])
                assert len(c["keep"]) == len(c["e"]), ln
            elif kind == "vote":
                c["counts"] = np.array(_ints(kv["counts"]), np.int64)
                c["n"] = int(kv["n"])
                c["rho"] = tuple(int(x) for x in kv["rho"].split("/"))
                c["keep"] = _digits(kv["keep"])
            elif kind == "runs":
                c["row"] = _digits(kv["row"])
                c["starts"] = _ints(kv["starts"])
                c["lens"] = _ints(kv["lens"])
            elif kind == "anchors":
                for key in ("F", "Hl", "Wl", "text", "stride"):
                    c[key] = int(kv[key])
                c["rows"] = _ints(kv["rows"])
                c["map"] = [tuple(int(y) for y in x.split(":")) for x in kv["map"].split(",")]
            else:
                raise ValueError(f"hand_worked.txt:{ln}: unknown case kind {kind!r}")
            cases[kind].append(c)
    return cases


def tiny_calibration():
    """The Tiny workload's oracle results, with masks and energies as numpy arrays."""
    with open(os.path.join(GOLDEN, "tiny_calibration.json")) as f:
        d = json.load(f)
    for sp in d["spaces"].values():
        shape = tuple(sp["shape"])
        sp["energy_f32"] = [np.array(w, np.uint32).view(np.float32).reshape(shape) for w in sp["energy_f32_bits"]]
        sp["mask_arrays"] = [_digits(m).reshape(shape) for m in sp["masks"]]
        sp["counts_array"] = np.array(sp["counts"], np.int64).reshape(shape)
        sp["vote_array"] = _digits(sp["vote"]).reshape(shape)
    w = d["workload"]
    sl = d["slice"]
    sl["mask_array"] = _digits(sl["mask"]).reshape(w["H"], w["nq"], w["nq"])
    at = d["attention"]
    at["O_array"] = np.array(at["O"], np.float64)
    at["LSE_array"] = np.array(at["LSE"], np.float64)
    return d
