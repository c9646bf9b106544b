"""The FMA-pipe exp2 of the energy pass (exp2_poly2 in csrc/ptx.cuh), checked on the CPU.

The coefficients in ptx.cuh must be the fp32 rounding of csrc/fit_exp2_poly.py's fit, and
the routine -- round-to-nearest reduction by adding 1.5 * 2^23, a degree-4 Horner chain of
fused multiply-adds, 2^n added to the exponent field as an integer -- is emulated in fp32
and compared with float64 2^x.  No GPU is needed."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "calibrated_block_sparse_calib_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _header_coefficients():
    """c0 .. c4 as written in exp2_poly2 (its Horner chain names c4 first, c0 last)."""
    src = open(os.path.join(CSRC, "ptx.cuh")).read()
    body = src[src.index("void exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    lits = [float(x) for x in re.findall(r"([0-9]+\.[0-9]+e-?[0-9]+|[0-9]+\.[0-9]+)f", body)]
    lits = [x for x in lits if x not in (12582912.0, 125.0, 127.0, 1.0)]
    uniq = []
    for x in lits:                      # each coefficient appears twice (packed pair)
        if not uniq or uniq[-1] != x:
            uniq.append(x)
    assert len(uniq) == 5, uniq
    c4, c3, c2, c1, c0 = uniq
    return np.array([c0, c1, c2, c3, c4], np.float32)


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _exp2_poly_emulated(x, c):
    """fp32 emulation of exp2_poly2 for one lane (inputs clamped to [-125, 127], as on the device)."""
    x = np.clip(x.astype(np.float32), np.float32(-125.0), np.float32(127.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    r = _fma32(n, np.full_like(n, -1.0), x)
    p = _fma32(np.full_like(r, c[4]), r, np.full_like(r, c[3]))
    for k in (2, 1, 0):
        p = _fma32(p, r, np.full_like(r, c[k]))
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))) % (1 << 32)
    return bits.astype(np.uint32).view(np.float32)


def test_header_coefficients_are_the_fit():
    fit = _fit_module()
    c = fit.fit().astype(np.float32)
    np.testing.assert_array_equal(_header_coefficients(), c)
    assert fit.max_rel_error(fit.fit()) < 3e-6


def test_exp2_poly_matches_exp2_over_its_range():
    c = _header_coefficients()
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.uniform(-125.0, 127.0, 200000), np.arange(-125, 127.25, 0.5),
                        rng.uniform(-1.0, 1.0, 20000)]).astype(np.float32)
    y = _exp2_poly_emulated(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 3e-6, float(rel.max())


def test_exp2_poly_clamps_below_and_masked_inputs():
    c = _header_coefficients()
    y = _exp2_poly_emulated(np.array([-np.inf, -1000.0, -126.0], np.float32), c).astype(np.float64)
    assert np.all(np.abs(y / 2.0 ** -125 - 1.0) < 3e-6)
