"""The pins discriminate: plausible mistakes planted in the oracle (on the CPU) make them fail.

Each test takes a pin used elsewhere -- a closed form, an invariant or a hand-worked case --
checks that the oracle satisfies it, then plants one mistake (a dropped scale, a transposed
operand or index, a dropped normalisation, an off-by-one, a flipped comparison or tie
order) in the oracle's code path and checks that the same pin now fails.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import oracle.calibatt_ref as ref
from golden_data import hand_worked

HW = hand_worked()


def _rand(seed, H, N, D):
    g = np.random.default_rng(seed)
    return [g.standard_normal((H, N, D)) for _ in range(3)]


def _sdpa(q, k, v, scale, allowed=None):
    """torch's scaled_dot_product_attention in float64 (the library routine the attention
    pins compare with); `allowed` is a boolean [Nq, N] token mask."""
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))
    mask = None if allowed is None else t(allowed)
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=mask, scale=scale).numpy()


def test_dense_pin_catches_a_dropped_scale(monkeypatch):
    q, k, v = _rand(1, 1, 200, 16)
    scale = 1 / math.sqrt(16)
    ones = np.ones((1, 4, 4), np.uint8)
    good, _ = oracle.sparse_attention(q, k, v, scale, 64, ones)
    assert np.allclose(good, _sdpa(q, k, v, scale), atol=1e-12)
    real = ref.logits
    monkeypatch.setattr(ref, "logits", lambda a, b, s: real(a, b, 1.0))
    bad, _ = oracle.sparse_attention(q, k, v, scale, 64, ones)
    assert not np.allclose(bad, _sdpa(q, k, v, scale), atol=1e-6)


def test_dense_pin_catches_transposed_logits(monkeypatch):
    # one 128-token block, so that K Q^T has the shape of Q K^T
    q, k, v = _rand(2, 1, 128, 16)
    scale = 0.25
    ones = np.ones((1, 1, 1), np.uint8)
    good, _ = oracle.sparse_attention(q, k, v, scale, 128, ones)
    assert np.allclose(good, _sdpa(q, k, v, scale), atol=1e-12)
    monkeypatch.setattr(ref, "logits", lambda a, b, s: (np.asarray(b, np.float64) @ np.asarray(a, np.float64).T) * s)
    bad, _ = oracle.sparse_attention(q, k, v, scale, 128, ones)
    assert not np.allclose(bad, _sdpa(q, k, v, scale), atol=1e-6)


def test_block_mask_pin_catches_a_transposed_mask():
    q, k, v = _rand(3, 1, 256, 8)
    B, scale = 64, 0.3
    m = np.array([[[1, 0, 0, 0], [1, 1, 0, 0], [0, 1, 1, 0], [1, 0, 1, 1]]], np.uint8)
    allowed = np.kron(m[0], np.ones((B, B))).astype(bool)
    good, _ = oracle.sparse_attention(q, k, v, scale, B, m)
    assert np.allclose(good, _sdpa(q, k, v, scale, allowed), atol=1e-12)
    bad, _ = oracle.sparse_attention(q, k, v, scale, B, np.swapaxes(m, 1, 2))
    assert not np.allclose(bad, _sdpa(q, k, v, scale, allowed), atol=1e-6)


def test_row_sum_pin_catches_a_dropped_normalisation():
    q, k, _ = _rand(4, 1, 192, 8)
    good = oracle.block_energy(q, k, 0.5, 64)
    rows = np.array([64.0, 64.0, 64.0])
    assert np.allclose(good.sum(axis=2)[0], rows)
    # P = exp(S) without the row LSE subtracted
    bad = oracle.block_energy(q, k, 0.5, 64, lse=np.zeros((1, 192)))
    assert not np.allclose(bad.sum(axis=2)[0], rows)


def test_anchor_pin_catches_a_dropped_stride(monkeypatch):
    case = HW["anchors"][0]
    F, Hl, Wl, S = case["F"], case["Hl"], case["Wl"], case["stride"]
    assert all(ref.anchor_token(t, F, Hl, Wl, S) == a for t, a in case["map"])

    def bad_anchor(t, F, Hl, Wl, stride):              # floor(y / s) without the * s
        nv = F * Hl * Wl
        if t >= nv:
            return t
        x, y, f = t % Wl, (t // Wl) % Hl, t // (Wl * Hl)
        return (f * Hl + y // stride) * Wl + x

    monkeypatch.setattr(ref, "anchor_token", bad_anchor)
    assert not all(ref.anchor_token(t, F, Hl, Wl, S) == a for t, a in case["map"])


def test_run_pin_catches_an_off_by_one_length(monkeypatch):
    case = HW["runs"][0]
    rp, ci = oracle.mask_to_csr(case["row"][None, None])
    real = ref.csr_to_intervals

    def bad(row_ptr, col_idx):
        ip, st, ln = real(row_ptr, col_idx)
        return ip, st, ln - 1
    monkeypatch.setattr(ref, "csr_to_intervals", bad)
    ip, st, ln = ref.csr_to_intervals(rp, ci)
    assert ln.tolist() != case["lens"]
    rp2, ci2 = oracle.intervals_to_csr(ip, st, ln)
    assert ci2.tolist() != ci.tolist()                  # the round trip breaks too


def test_vote_pin_catches_at_least_instead_of_above():
    case = next(c for c in HW["vote"] if c["counts"].tolist() == [2, 2, 1, 0])
    good = oracle.aggregate_masks(case["counts"][None, None], case["n"], *case["rho"])[0, 0]
    np.testing.assert_array_equal(good, case["keep"])
    # ">=" keeps the 2/4 blocks that the strict vote drops
    c, n, (num, den) = case["counts"], case["n"], case["rho"]
    bad = (c * den >= num * n).astype(np.uint8)
    assert not np.array_equal(bad, case["keep"])


def test_tie_pin_catches_ties_to_the_higher_index(monkeypatch):
    case = next(c for c in HW["select"] if c["e"].tolist() == [0.25] * 4 and c["tau"] == 0.5)
    np.testing.assert_array_equal(oracle.select_row(case["e"], case["tau"], case["diag"]).astype(np.uint8),
                                  case["keep"])
    real_sorted = sorted

    def sorted_high_first(it, key=None, reverse=False):
        # the oracle's order key is (not forced, -q, j); flip j to take higher indices first
        if key is not None:
            return real_sorted(it, key=lambda j: (key(j)[0], key(j)[1], -key(j)[2]), reverse=reverse)
        return real_sorted(it, reverse=reverse)
    monkeypatch.setattr(ref, "sorted", sorted_high_first, raising=False)
    bad = oracle.select_row(case["e"], case["tau"], case["diag"]).astype(np.uint8)
    assert not np.array_equal(bad, case["keep"])


def test_repeat_similarity_pin_catches_a_wrong_pairing(monkeypatch):
    """Member queries equal to their anchors' give cosine 1 (pin); pairing each token with
    the wrong row breaks it."""
    F, Hl, Wl, s = 1, 4, 4, 2
    rng = np.random.default_rng(9)
    q = rng.standard_normal((1, 16, 8))
    k = rng.standard_normal((1, 16, 8))
    for t in range(16):
        q[0, t] = q[0, ref.anchor_token(t, F, Hl, Wl, s)]
    members = [5, 6, 13, 14]                            # odd latent rows: not their own anchor
    good = oracle.repeat_similarity(q, k, 0.5, members, F, Hl, Wl, s)
    assert np.allclose(good, 1.0)
    monkeypatch.setattr(ref, "anchor_token", lambda t, F, Hl, Wl, stride: (t + 1) % (F * Hl * Wl))
    bad = ref.repeat_similarity(q, k, 0.5, members, F, Hl, Wl, s)
    assert not np.allclose(bad, 1.0)
