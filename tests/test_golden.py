"""The oracle against the fixtures under tests/golden/ (CPU).

hand_worked.txt: cases derived by hand from the pages' rules (minimal tau-selection, the
vote, skip-list runs, anchor rows) with exact dyadic energies -- a pin independent of the
oracle's code.  tiny_calibration.json: the oracle's own results for the Tiny workload,
written by tests/golden/make_tiny_golden.py; checking that the oracle still reproduces
them makes any change to its arithmetic visible (such a change must cite the passage that
justifies it), and the GPU tests compare the kernels with the stored values.
"""
import math

import numpy as np
import pytest

import oracle
from golden_data import hand_worked, tiny_calibration

HW = hand_worked()


@pytest.mark.parametrize("case", HW["select"], ids=lambda c: f"line{c['line']}")
def test_hand_worked_select(case):
    keep = oracle.select_row(case["e"], case["tau"], case["diag"], case["forced"])
    np.testing.assert_array_equal(keep.astype(np.uint8), case["keep"])


@pytest.mark.parametrize("case", HW["vote"], ids=lambda c: f"line{c['line']}")
def test_hand_worked_vote(case):
    keep = oracle.aggregate_masks(case["counts"][None, None], case["n"], *case["rho"])
    np.testing.assert_array_equal(keep[0, 0], case["keep"])


@pytest.mark.parametrize("case", HW["runs"], ids=lambda c: f"line{c['line']}")
def test_hand_worked_runs(case):
    rp, ci = oracle.mask_to_csr(case["row"][None, None])
    ip, st, ln = oracle.csr_to_intervals(rp, ci)
    assert st.tolist() == case["starts"] and ln.tolist() == case["lens"]
    assert ip.tolist() == [0, len(case["starts"])]


@pytest.mark.parametrize("case", HW["anchors"], ids=lambda c: f"line{c['line']}")
def test_hand_worked_anchors(case):
    rows = oracle.anchor_rows(case["F"], case["Hl"], case["Wl"], case["text"], case["stride"])
    assert rows.tolist() == case["rows"]
    for t, a in case["map"]:
        assert oracle.anchor_token(t, case["F"], case["Hl"], case["Wl"], case["stride"]) == a
        # the compacted index the token reads its output from holds that anchor
        idx = oracle.anchor_index_of_token(t, case["F"], case["Hl"], case["Wl"], case["text"], case["stride"])
        assert rows[idx] == a


def test_hand_worked_file_covers_every_kind():
    assert len(HW["select"]) >= 20 and len(HW["vote"]) >= 5
    assert len(HW["runs"]) >= 5 and len(HW["anchors"]) >= 2


# ------------------------------------------------------------------------------------
# Tiny workload: the oracle reproduces its stored results
# ------------------------------------------------------------------------------------

@pytest.fixture(scope="module")
def tiny():
    return tiny_calibration()


def test_tiny_inputs_unchanged(tiny):
    from golden.make_tiny_golden import input_digest
    from calibrated_block_sparse_calib_b200 import synth
    wl = synth.WORKLOADS["tiny"]
    for d, want in enumerate(tiny["inputs_sha256"]):
        assert input_digest(*synth.make_qkv(wl, input_idx=d)) == want


def test_tiny_selection_and_vote_from_stored_energies(tiny):
    """Selection is bit-exact from identical float32 energies: the stored masks follow from
    the stored energies, and the vote from the masks."""
    w = tiny["workload"]
    for sp in tiny["spaces"].values():
        counts = np.zeros_like(sp["counts_array"])
        for e32, m in zip(sp["energy_f32"], sp["mask_arrays"]):
            got = oracle.select_mask(e32, w["tau"])
            np.testing.assert_array_equal(got, m)
            counts += got
        np.testing.assert_array_equal(counts, sp["counts_array"])
        np.testing.assert_array_equal(oracle.aggregate_masks(counts, w["n_inputs"], *w["rho"]), sp["vote_array"])


def test_tiny_slice_lists(tiny):
    w = tiny["workload"]
    sl = tiny["slice"]
    m = sl["mask_array"]
    for h in range(w["H"]):
        sp = tiny["spaces"]["anchor" if w["repeat"][h] else "full"]["vote_array"][h]
        np.testing.assert_array_equal(m[h, :sp.shape[0]], sp)
        assert not m[h, sp.shape[0]:].any()
    rp, ci = oracle.mask_to_csr(m)
    assert rp.tolist() == sl["row_ptr"] and ci.tolist() == sl["col_idx"]
    assert oracle.build_schedule(rp, w["H"], w["nq"]).tolist() == sl["work"]


def test_tiny_oracle_recomputes_the_fixture(tiny):
    """Energies to within 4 float32 ulps (BLAS may order a dot product differently on
    another machine), attention rows to 1e-12."""
    from golden.make_tiny_golden import compute
    doc = compute()
    for name, sp in tiny["spaces"].items():
        for a, b in zip(doc["spaces"][name]["energy_f32_bits"], sp["energy_f32_bits"]):
            fa = np.array(a, np.uint32).view(np.float32).astype(np.float64)
            fb = np.array(b, np.uint32).view(np.float32).astype(np.float64)
            assert np.all(np.abs(fa - fb) <= 4 * np.spacing(np.abs(fb).astype(np.float32)).astype(np.float64))
    np.testing.assert_allclose(np.array(doc["attention"]["O"]), tiny["attention"]["O_array"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(np.array(doc["attention"]["LSE"]), tiny["attention"]["LSE_array"], rtol=0,
                               atol=1e-12)
    assert doc["slice"]["mask"] == tiny["slice"]["mask"]


def test_tiny_fixture_invariants(tiny):
    """Properties the pages fix, read off the stored values: every row's energies sum to
    its query-row count (softmax rows sum to 1), every kept set reaches tau and has no
    redundant block, and rows of the repeat head equal their anchor's output."""
    w = tiny["workload"]
    B, N = w["block"], w["N"]
    for name, sp in tiny["spaces"].items():
        Nq = N if name == "full" else w["n_anchor"]
        nq = sp["energy_f32"][0].shape[1]
        rows = np.array([min((i + 1) * B, Nq) - i * B for i in range(nq)], np.float64)
        for e32, m in zip(sp["energy_f32"], sp["mask_arrays"]):
            e = e32.astype(np.float64)
            np.testing.assert_allclose(e.sum(axis=2), np.broadcast_to(rows, e.shape[:2]), rtol=1e-6)
            kept = (e * m).sum(axis=2)
            assert np.all(kept >= w["tau"] * e.sum(axis=2) * (1 - 1e-6))
            # dropping the smallest kept block falls below tau
            smallest = np.where(m > 0, e, np.inf).min(axis=2)
            assert np.all(kept - smallest < w["tau"] * e.sum(axis=2) * (1 + 1e-6))
    at = tiny["attention"]
    rows = at["rows"]
    O = at["O_array"]
    for h, rep in enumerate(w["repeat"]):
        if not rep:
            continue
        for n, t in enumerate(rows):
            a = oracle.anchor_token(t, w["F"], w["Hl"], w["Wl"], w["stride"])
            if a in rows:
                np.testing.assert_array_equal(O[h, n], O[h, rows.index(a)])
    assert np.all(np.isfinite(O)) and math.isfinite(float(at["LSE_array"].max()))
