"""Pins for the oracle's logits / LSE / block-energy functions (CPU only).

Each pin comes from something other than the oracle itself: closed forms implied by
the definition (rows of a softmax sum to one; a constant logit row is uniform),
brute force with scipy's softmax and explicit index loops, and scipy's logsumexp.
"""
import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle
from conftest import to64


def _rand(H, N, D, seed):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((H, N, D)), rng.standard_normal((H, N, D))


@pytest.mark.parametrize("N,B", [(512, 64), (300, 64), (130, 128), (64, 64), (7, 64)])
def test_energy_row_sums_equal_block_rows(N, B):
    # P rows sum to 1, so sum_j E[i, j] = |I_i| exactly (up to rounding).
    q, k = _rand(2, N, 16, 1)
    q *= 2.0  # sharper rows
    E = oracle.block_energy(q, k, 0.25, B)
    nq = -(-N // B)
    sizes = np.array([min((i + 1) * B, N) - i * B for i in range(nq)], float)
    np.testing.assert_allclose(E.sum(axis=2), np.broadcast_to(sizes, (2, nq)), rtol=1e-12)


@pytest.mark.parametrize("N,B", [(512, 64), (300, 64), (200, 128)])
def test_energy_uniform_when_q_zero(N, B):
    # Q = 0 -> S = 0 -> P = 1/N everywhere -> E[i, j] = |I_i| |J_j| / N.
    _, k = _rand(1, N, 8, 2)
    q = np.zeros_like(k)
    E = oracle.block_energy(q, k, 0.3, B)
    n = -(-N // B)
    sz = np.array([min((i + 1) * B, N) - i * B for i in range(n)], float)
    np.testing.assert_allclose(E[0], np.outer(sz, sz) / N, rtol=1e-13)


def test_energy_uniform_when_keys_equal():
    # all keys equal -> each logit row is constant -> uniform P.
    N, B = 256, 64
    q, _ = _rand(1, N, 8, 3)
    k = np.tile(np.random.default_rng(4).standard_normal((1, 1, 8)), (1, N, 1))
    E = oracle.block_energy(q, k, 0.7, B)
    np.testing.assert_allclose(E[0], np.full((4, 4), B * B / N), rtol=1e-12)


def test_energy_brute_force_tiny(tiny_inputs):
    # Materialise P with scipy's softmax and sum each block with explicit loops.
    wl, qkv = tiny_inputs
    q, k, _ = (to64(t) for t in qkv[0])
    B, D = wl.shape.block, wl.shape.D
    scale = 1.0 / np.sqrt(D)
    E = oracle.block_energy(q, k, scale, B)
    H, N, _ = q.shape
    nb = N // B
    for h in range(H):
        P = softmax(scale * np.einsum("rd,cd->rc", q[h], k[h]), axis=1)
        ref = np.zeros((nb, nb))
        for r in range(N):
            for j in range(nb):
                ref[r // B, j] += P[r, j * B:(j + 1) * B].sum()
        np.testing.assert_allclose(E[h], ref, rtol=1e-11, atol=1e-300)


def test_row_lse_matches_scipy(tiny_inputs):
    wl, qkv = tiny_inputs
    q, k, _ = (to64(t) for t in qkv[1])
    scale = 1.0 / np.sqrt(wl.shape.D)
    L = oracle.row_lse(q, k, scale)
    for h in range(q.shape[0]):
        ref = logsumexp(scale * np.einsum("rd,cd->rc", q[h], k[h]), axis=1)
        np.testing.assert_allclose(L[h], ref, rtol=1e-13)


def test_cached_lse_and_subsets_agree(tiny_inputs):
    wl, qkv = tiny_inputs
    q, k, _ = (to64(t) for t in qkv[2])
    B = wl.shape.block
    scale = 1.0 / np.sqrt(wl.shape.D)
    E = oracle.block_energy(q, k, scale, B)
    L = oracle.row_lse(q, k, scale)
    np.testing.assert_allclose(oracle.block_energy(q, k, scale, B, lse=L), E, rtol=1e-12)
    sub = oracle.block_energy(q, k, scale, B, q_blocks=[5, 1])
    np.testing.assert_allclose(sub, E[:, [5, 1]], rtol=1e-13)
    # q_rows = a permutation-free subset: energies of the gathered rows match a direct
    # computation on the gathered tensor.
    rows = np.arange(0, q.shape[1], 2)
    Eg = oracle.block_energy(q, k, scale, B, q_rows=rows)
    Ed = oracle.block_energy(q[:, rows], k, scale, B)
    np.testing.assert_allclose(Eg, Ed, rtol=1e-13)


def test_energy_mean_single_input_identity():
    e = np.random.default_rng(5).random((2, 3, 4)).astype(np.float32)
    np.testing.assert_array_equal(oracle.energy_mean([e]), e)
    m = oracle.energy_mean([e, 3 * e])
    np.testing.assert_allclose(m, (2 * e.astype(np.float64)).astype(np.float32), rtol=0)


def test_energy_mean_rows_sum_to_one_softmax_row_per_query():
    """Each input's query rows sum to one softmax row each (sum_j E[i, j] = |I_i|), so the
    mean over inputs keeps that sum; the plain sum over three inputs (the 1/D_cal factor
    dropped) would give 3 |I_i| and fails this pin."""
    Es = []
    for seed in (11, 12, 13):
        q, k = _rand(1, 200, 8, seed)
        Es.append(oracle.block_energy(q, k, 0.7, 64))
    rows = np.array([64, 64, 64, 8], np.float64)
    mean = oracle.energy_mean(Es).astype(np.float64)
    np.testing.assert_allclose(mean.sum(axis=2)[0], rows, rtol=1e-6)
    assert not np.allclose(sum(Es).sum(axis=2)[0], rows, rtol=1e-3)


def test_row_sum_pin_catches_a_mean_instead_of_a_sum(monkeypatch):
    # Plant a plausible mistake in the oracle (block mean instead of block sum) and
    # check the row-sum pin fails: the pins discriminate.
    q, k = _rand(1, 256, 8, 9)
    good = oracle.block_energy(q, k, 0.5, 64)
    bad = good / (64.0 * 64.0)
    assert np.allclose(good.sum(axis=2), 64.0)
    assert not np.allclose(bad.sum(axis=2), 64.0)
    # A transposed block index (E[j, i]) breaks it too for non-symmetric inputs.
    assert not np.allclose(np.swapaxes(good, 1, 2).sum(axis=2), 64.0)
