"""Pins for the oracle's interval form of skip lists (CPU).

Independent references: the number of runs in a mask row equals its 0 -> 1 transitions
(numpy diff of the padded row); a hand-worked row; decode(encode(x)) == x; runs are maximal
(no two consecutive runs touch) and strictly ascending; empty and full rows.
"""
import numpy as np
import pytest

import oracle


def test_hand_worked_row():
    m = np.array([[[1, 1, 0, 1, 0, 0, 1, 1, 1]]], np.uint8)
    rp, ci = oracle.mask_to_csr(m)
    ip, st, ln = oracle.csr_to_intervals(rp, ci)
    assert ip.tolist() == [0, 3]
    assert st.tolist() == [0, 3, 6] and ln.tolist() == [2, 1, 3]


@pytest.mark.parametrize("seed,p", [(1, 0.1), (2, 0.5), (3, 0.9)])
def test_run_count_equals_rising_edges_and_round_trip(seed, p):
    rng = np.random.default_rng(seed)
    H, nq, nk = 3, 9, 70
    m = (rng.random((H, nq, nk)) < p).astype(np.uint8)
    m[0, 0] = 0          # an empty row
    m[1, 1] = 1          # a full row
    rp, ci = oracle.mask_to_csr(m)
    ip, st, ln = oracle.csr_to_intervals(rp, ci)
    flat = m.reshape(H * nq, nk).astype(np.int64)
    rises = (np.diff(np.pad(flat, ((0, 0), (1, 0))), axis=1) == 1).sum(axis=1)
    np.testing.assert_array_equal(np.diff(ip), rises)
    assert ip.dtype == np.int32 and st.dtype == np.int16 and ln.dtype == np.int16
    assert ip[1] - ip[0] == 0                      # empty row: no run
    r_full = 1 * nq + 1
    assert ip[r_full + 1] - ip[r_full] == 1 and st[ip[r_full]] == 0 and ln[ip[r_full]] == nk
    for r in range(H * nq):
        s_, l_ = st[ip[r]:ip[r + 1]].astype(np.int64), ln[ip[r]:ip[r + 1]].astype(np.int64)
        assert np.all(l_ >= 1)
        assert np.all(s_[1:] > s_[:-1] + l_[:-1])   # maximal: a gap between runs
    rp2, ci2 = oracle.intervals_to_csr(ip, st, ln)
    np.testing.assert_array_equal(rp2, rp)
    np.testing.assert_array_equal(ci2, ci)


def test_band_mask_compresses_to_one_run_per_row():
    nq = nk = 20
    m = np.zeros((1, nq, nk), np.uint8)
    for i in range(nq):
        m[0, i, max(0, i - 3):min(nk, i + 4)] = 1
    rp, ci = oracle.mask_to_csr(m)
    ip, st, ln = oracle.csr_to_intervals(rp, ci)
    assert np.all(np.diff(ip) == 1)
    assert int(ln.astype(np.int64).sum()) == int(m.sum())
