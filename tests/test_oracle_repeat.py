"""Pins for the oracle's spatial-repetition detection (CPU).

Independent references: scipy's cosine distance on a softmax computed by scipy; a head
whose member queries equal their anchors' queries (cosine 1, flagged for any gamma < 1); a
head whose keys give every query row a one-hot softmax on a different key (cosine 0);
anchors compared with themselves; and the mean excluding tokens that are their own anchor.
"""
import numpy as np
from scipy.spatial.distance import cosine
from scipy.special import softmax

import oracle

F, HL, WL, S_ = 3, 8, 5, 4


def _members(rng, n):
    return rng.integers(0, F * HL * WL, size=n)


def test_matches_scipy_cosine_of_scipy_softmax():
    rng = np.random.default_rng(0)
    N, D = F * HL * WL, 16
    q, k = rng.standard_normal((2, N, D)), rng.standard_normal((2, N, D))
    mem = _members(rng, 25)
    sim = oracle.repeat_similarity(q, k, 0.3, mem, F, HL, WL, S_)
    for h in range(2):
        P = softmax(0.3 * q[h] @ k[h].T, axis=1)
        for i, b in enumerate(mem):
            a = oracle.anchor_token(int(b), F, HL, WL, S_)
            assert abs(sim[h, i] - (1.0 - cosine(P[a], P[b]))) < 1e-12


def test_anchor_token_definition():
    # (f, y, x) -> (f, floor(y/4)*4, x); text tokens are their own anchor
    assert oracle.anchor_token((1 * HL + 7) * WL + 3, F, HL, WL, 4) == (1 * HL + 4) * WL + 3
    assert oracle.anchor_token((2 * HL + 4) * WL + 0, F, HL, WL, 4) == (2 * HL + 4) * WL + 0
    assert oracle.anchor_token(F * HL * WL + 2, F, HL, WL, 4) == F * HL * WL + 2


def test_identical_queries_give_one_and_flag():
    rng = np.random.default_rng(1)
    N, D = F * HL * WL, 8
    k = rng.standard_normal((1, N, D))
    q = rng.standard_normal((1, N, D))
    for t in range(N):
        q[0, t] = q[0, oracle.anchor_token(t, F, HL, WL, S_)]
    mem = _members(rng, 40)
    sim = oracle.repeat_similarity(q, k, 0.5, mem, F, HL, WL, S_)
    np.testing.assert_allclose(sim, 1.0, atol=1e-12)
    mean, flag = oracle.repeat_flags(sim, mem, F, HL, WL, S_, 0.999)
    assert flag[0] and abs(mean[0] - 1) < 1e-12


def test_disjoint_one_hot_rows_give_zero():
    # key c is aligned with query direction c only: each row's softmax is ~one-hot on its
    # own key, so a member and its (different) anchor have disjoint support
    N = F * HL * WL
    q = np.eye(N)[None] * 60.0
    k = np.eye(N)[None]
    mem = np.array([t for t in range(N) if oracle.anchor_token(t, F, HL, WL, S_) != t][:30])
    sim = oracle.repeat_similarity(q, k, 1.0, mem, F, HL, WL, S_)
    assert np.all(np.abs(sim) < 1e-20)
    mean, flag = oracle.repeat_flags(sim, mem, F, HL, WL, S_, 0.5)
    assert not flag[0] and mean[0] < 1e-20


def test_mean_excludes_tokens_that_are_their_own_anchor():
    mem = np.array([0, WL, 2 * WL])              # rows y = 0 (anchor), 1, 2 of frame 0
    sim = np.array([[1.0, 0.25, 0.5]])           # exact binary fractions
    mean, flag = oracle.repeat_flags(sim, mem, F, HL, WL, S_, 0.3)
    assert mean[0] == 0.375 and flag[0]
    mean, flag = oracle.repeat_flags(sim, mem, F, HL, WL, S_, 0.375)
    assert not flag[0]                            # "exceeds": strict
