"""Pins for the oracle's minimal tau-energy selection and the cross-input vote (CPU).

Pins: the defining invariant (the kept prefix reaches T, the prefix one shorter does
not), brute force over all 2^nk subsets, hand-worked rows, and special cases
(tau -> 0+, one-hot, uniform, tau = 1, all-zero rows, forced blocks).
"""
import itertools
import math

import numpy as np
import pytest

import oracle


def _threshold(q, tau):
    Q = int(sum(int(x) for x in q))
    return max(1, math.ceil(float(np.float64(tau) * np.float64(Q)))), Q


def _rows(seed, n, nk):
    rng = np.random.default_rng(seed)
    out = []
    for t in range(n):
        kind = t % 5
        if kind == 0:
            e = rng.random(nk)
        elif kind == 1:
            e = rng.exponential(size=nk) ** 4
        elif kind == 2:
            e = np.round(rng.random(nk) * 4) / 4           # many exact ties
        elif kind == 3:
            e = np.exp(-30 * rng.random(nk))               # wide dynamic range
        else:
            e = rng.random(nk) * 1e-30                     # tiny magnitudes
        out.append(e.astype(np.float32))
    return out


@pytest.mark.parametrize("nk", [1, 2, 7, 8, 33, 256, 591])
@pytest.mark.parametrize("tau", [1e-6, 0.5, 0.9, 0.95, 0.99, 1.0])
def test_kept_prefix_reaches_tau_and_is_minimal(nk, tau):
    for r, e in enumerate(_rows(nk * 7 + int(tau * 100), 10, nk)):
        keep = oracle.select_row(e, tau, r % nk)
        q, _ = oracle.quantize_row(e)
        T, Q = _threshold(q, tau)
        if Q == 0:                      # all-zero row: the diagonal (or block 0) alone
            assert keep.sum() == 1 and keep[(r % nk) if (r % nk) < nk else 0]
            continue
        assert T <= Q
        kept = sorted((int(q[j]) for j in np.nonzero(keep)[0]), reverse=True)
        # reaches: sum >= T; minimal: dropping the smallest kept block falls below T
        assert sum(kept) >= T
        assert sum(kept) - kept[-1] < T
        # the kept blocks are the largest ones: nothing dropped beats a kept block
        dropped = [int(q[j]) for j in np.nonzero(~keep)[0]]
        if dropped:
            assert max(dropped) <= kept[-1]


def test_brute_force_minimum_cardinality_nk8():
    rng = np.random.default_rng(11)
    for t in range(60):
        e = (rng.random(8) ** (1 + t % 4)).astype(np.float32)
        if t % 7 == 0:
            e[rng.integers(0, 8)] = e.max()                # force a tie at the top
        tau = [0.5, 0.8, 0.9, 0.95, 0.99][t % 5]
        keep = oracle.select_row(e, tau, t % 8)
        q, _ = oracle.quantize_row(e)
        T, _ = _threshold(q, tau)
        best = None
        best_sum = -1
        for size in range(1, 9):
            for sub in itertools.combinations(range(8), size):
                s = sum(int(q[j]) for j in sub)
                if s >= T:
                    best = size if best is None else best
                    if size == best:
                        best_sum = max(best_sum, s)
            if best is not None:
                break
        assert keep.sum() == best
        assert sum(int(q[j]) for j in np.nonzero(keep)[0]) == best_sum


def test_hand_worked_rows():
    # Energies 0.05, 0.5, 0.15, 0.3 with tau = 0.9: sorted 0.5, 0.3, 0.15 reach
    # 0.95 >= 0.9 of the total 1.0 after three blocks; two (0.8) do not.
    e = np.array([0.05, 0.5, 0.15, 0.3], np.float32)
    np.testing.assert_array_equal(oracle.select_row(e, 0.9, 0), [0, 1, 1, 1])
    # tau = 0.45: the single largest block (0.5 of 1.0) reaches it.  (tau = 0.5 would sit
    # on the boundary: the float32 images of 0.05, 0.15, 0.3 sum to slightly above 0.5.)
    np.testing.assert_array_equal(oracle.select_row(e, 0.45, 0), [0, 1, 0, 0])
    # tau = 0.51: needs the two largest.
    np.testing.assert_array_equal(oracle.select_row(e, 0.51, 0), [0, 1, 0, 1])
    # equal energies: ties go to the lower key index.
    e2 = np.array([0.25, 0.25, 0.25, 0.25], np.float32)
    np.testing.assert_array_equal(oracle.select_row(e2, 0.5, 3), [1, 1, 0, 0])


def test_special_cases():
    rng = np.random.default_rng(3)
    e = rng.random(50).astype(np.float32)
    # tau -> 0+: only the argmax block
    keep = oracle.select_row(e, 1e-12, 0)
    assert keep.sum() == 1 and keep[int(np.argmax(e))]
    # one-hot energy: one block whatever tau
    oh = np.zeros(50, np.float32)
    oh[17] = 3.0
    for tau in (0.1, 0.99, 1.0):
        keep = oracle.select_row(oh, tau, 0)
        assert keep.sum() == 1 and keep[17]
    # uniform energy: ceil(tau * nk) blocks (tau * nk away from an integer)
    u = np.full(40, 0.125, np.float32)
    for tau in (0.33, 0.5 + 1e-3, 0.9, 0.951):
        assert oracle.select_row(u, tau, 0).sum() == math.ceil(tau * 40)
    # tau = 1: exactly the blocks with non-zero quantised energy
    z = e.copy()
    z[::3] = 0.0
    keep = oracle.select_row(z, 1.0, 0)
    q, _ = oracle.quantize_row(z)
    np.testing.assert_array_equal(keep, q > 0)
    # all-zero row keeps the diagonal block, or block 0 past the end
    np.testing.assert_array_equal(np.nonzero(oracle.select_row(np.zeros(9, np.float32), 0.9, 4))[0], [4])
    np.testing.assert_array_equal(np.nonzero(oracle.select_row(np.zeros(9, np.float32), 0.9, 12))[0], [0])


def test_forced_blocks_are_kept_and_count_toward_tau():
    rng = np.random.default_rng(8)
    for t in range(40):
        nk = 12
        e = rng.random(nk).astype(np.float32)
        forced = rng.random(nk) < 0.25
        tau = 0.9
        keep = oracle.select_row(e, tau, 0, forced)
        assert keep[forced].all()
        q, _ = oracle.quantize_row(e)
        T, _ = _threshold(q, tau)
        free = [int(q[j]) for j in np.nonzero(keep & ~forced)[0]]
        total = int(sum(int(q[j]) for j in np.nonzero(keep)[0]))
        assert total >= T
        if free:                       # the free part is minimal
            assert total - min(free) < T


def test_quantisation_is_exact_and_monotone():
    for e in _rows(21, 25, 591):
        q, Q = oracle.quantize_row(e)
        nk = len(e)
        c = oracle.ceil_log2(nk)
        assert Q < 2 ** 53
        assert int(q.max()) <= 2 ** (52 - c)
        assert float(np.sum(q.astype(np.float64))) == float(Q)   # float64 sum is exact
        order = np.argsort(e, kind="stable")
        assert np.all(np.diff(q[order].astype(np.int64)) >= 0)


def test_aggregation_vote():
    rng = np.random.default_rng(2)
    m = (rng.random((2, 5, 6)) < 0.4).astype(np.uint8)
    m[:, :, 0] = 1
    # one input, rho = 1/2: the vote is the identity
    np.testing.assert_array_equal(oracle.aggregate_masks(m.astype(np.int32), 1, 1, 2), m)
    # three inputs, rho = 1/2: majority (count >= 2)
    counts = rng.integers(0, 4, size=(2, 5, 6)).astype(np.int32)
    counts[:, :, 1] = 3
    agg = oracle.aggregate_masks(counts, 3, 1, 2)
    np.testing.assert_array_equal(agg, (counts >= 2).astype(np.uint8))
    # strictness: with 4 inputs and rho = 1/2, count 2 is not above half
    c4 = np.array([[[2, 3, 1, 4]]], np.int32)
    np.testing.assert_array_equal(oracle.aggregate_masks(c4, 4, 1, 2), [[[0, 1, 0, 1]]])
    # a row the vote empties keeps its most frequent block (lowest index on ties)
    c = np.array([[[1, 2, 2, 0]]], np.int32)
    np.testing.assert_array_equal(oracle.aggregate_masks(c, 5, 1, 2), [[[0, 1, 0, 0]]])


def test_minimality_pin_catches_a_strict_comparison():
    # Plant a mistake: stop only when the prefix is strictly above T.  The minimality
    # pin must reject it on a row where some prefix lands exactly on T.
    e = np.array([0.5, 0.25, 0.25, 0.0], np.float32)
    q, _ = oracle.quantize_row(e)
    T, _ = _threshold(q, 0.75)
    good = oracle.select_row(e, 0.75, 0)
    bad = good.copy()
    bad[2] = True                                  # what ">" would keep
    for keep, ok in ((good, True), (bad, False)):
        kept = sorted((int(q[j]) for j in np.nonzero(keep)[0]), reverse=True)
        assert (sum(kept) >= T and sum(kept) - kept[-1] < T) == ok
