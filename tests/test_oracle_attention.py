"""Pins for the oracle's sparse attention, spatial repetition, skip lists and schedule (CPU).

Independent references: torch's scaled_dot_product_attention in float64 on CPU (with
an explicit token-level boolean mask built by np.kron from the block mask), scipy's
softmax / logsumexp, and closed forms (constant V, masked blocks contribute zero,
non-anchor rows equal their anchor, stride 1 equals plain attention).
"""
import numpy as np
import pytest
import torch
from scipy.special import logsumexp, softmax

import oracle
from conftest import to64


def _qkv(H, N, D, seed, scale_pos=1.0):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((H, N, D)) * scale_pos for _ in range(3)]


def _token_mask(block_mask, B, Nq, N):
    m = np.kron(block_mask.astype(bool), np.ones((B, B), bool))
    return m[:Nq, :N]


def _sdpa(q, k, v, scale, tok_mask=None):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    am = None if tok_mask is None else t(tok_mask)
    return torch.nn.functional.scaled_dot_product_attention(
        t(q)[None], t(k)[None], t(v)[None], attn_mask=am, scale=scale)[0].numpy()


@pytest.mark.parametrize("N,B", [(512, 64), (300, 64), (200, 128), (33, 64)])
def test_all_kept_equals_dense_sdpa(N, B):
    q, k, v = _qkv(2, N, 16, N)
    nb = -(-N // B)
    O, L = oracle.sparse_attention(q, k, v, 0.25, B, np.ones((2, nb, nb), np.uint8))
    np.testing.assert_allclose(O, _sdpa(q, k, v, 0.25), rtol=1e-11, atol=1e-12)
    for h in range(2):
        np.testing.assert_allclose(L[h], logsumexp(0.25 * q[h] @ k[h].T, axis=1), rtol=1e-13)


@pytest.mark.parametrize("N,B", [(512, 64), (300, 64)])
def test_block_mask_equals_token_mask_sdpa(N, B):
    q, k, v = _qkv(2, N, 16, 3)
    nb = -(-N // B)
    rng = np.random.default_rng(4)
    mask = (rng.random((2, nb, nb)) < 0.4).astype(np.uint8)
    mask[:, np.arange(nb), np.arange(nb)] = 1
    O, _ = oracle.sparse_attention(q, k, v, 0.3, B, mask)
    for h in range(2):
        ref = _sdpa(q[h:h + 1], k[h:h + 1], v[h:h + 1], 0.3, _token_mask(mask[h], B, N, N)[None])
        np.testing.assert_allclose(O[h], ref[0], rtol=1e-11, atol=1e-12)


def test_masked_blocks_contribute_exactly_zero():
    N, B = 320, 64
    q, k, v = _qkv(1, N, 8, 5)
    nb = 5
    mask = np.zeros((1, nb, nb), np.uint8)
    mask[0, :, [0, 2]] = 1
    O, L = oracle.sparse_attention(q, k, v, 0.5, B, mask)
    k2, v2 = k.copy(), v.copy()
    rng = np.random.default_rng(6)
    for j in (1, 3, 4):
        k2[0, j * B:(j + 1) * B] = rng.standard_normal((B, 8)) * 10
        v2[0, j * B:(j + 1) * B] = rng.standard_normal((B, 8)) * 10
    O2, L2 = oracle.sparse_attention(q, k2, v2, 0.5, B, mask)
    np.testing.assert_array_equal(O, O2)
    np.testing.assert_array_equal(L, L2)


def test_single_kept_block_is_softmax_over_its_keys():
    N, B = 256, 64
    q, k, v = _qkv(1, N, 8, 7)
    mask = np.zeros((1, 4, 4), np.uint8)
    mask[0, :, 2] = 1
    O, _ = oracle.sparse_attention(q, k, v, 0.4, B, mask)
    P = softmax(0.4 * q[0] @ k[0, 128:192].T, axis=1)
    np.testing.assert_allclose(O[0], P @ v[0, 128:192], rtol=1e-12, atol=1e-13)


def test_constant_v_gives_constant_output():
    N, B = 200, 64
    q, k, _ = _qkv(1, N, 8, 8)
    c = np.random.default_rng(9).standard_normal(8)
    v = np.tile(c, (1, N, 1))
    mask = (np.random.default_rng(10).random((1, 4, 4)) < 0.5).astype(np.uint8)
    mask[0, :, 0] = 1
    O, _ = oracle.sparse_attention(q, k, v, 0.4, B, mask)
    np.testing.assert_allclose(O[0], np.tile(c, (N, 1)), rtol=1e-13, atol=1e-14)


def test_empty_row_outputs_zero():
    q, k, v = _qkv(1, 128, 8, 11)
    mask = np.ones((1, 2, 2), np.uint8)
    mask[0, 1] = 0
    O, L = oracle.sparse_attention(q, k, v, 0.4, 64, mask)
    assert np.all(O[0, 64:] == 0) and np.all(np.isneginf(L[0, 64:]))
    assert np.all(np.isfinite(O[0, :64]))


def test_anchor_rows_and_inverse_map():
    for F, Hl, Wl, nt, s in [(4, 8, 16, 0, 2), (3, 45, 5, 0, 4), (2, 30, 7, 16, 4), (2, 5, 3, 4, 1)]:
        A = oracle.anchor_rows(F, Hl, Wl, nt, s)
        assert len(A) == F * (-(-Hl // s)) * Wl + nt
        N = F * Hl * Wl + nt
        for a, t in enumerate(A):
            assert oracle.anchor_index_of_token(int(t), F, Hl, Wl, nt, s) == a
        for t in range(N):
            a = oracle.anchor_index_of_token(t, F, Hl, Wl, nt, s)
            ta = int(A[a])
            if t >= F * Hl * Wl:
                assert ta == t
            else:  # same frame, same column, anchor row = floor(y/s)*s
                assert ta // (Hl * Wl) == t // (Hl * Wl) and ta % Wl == t % Wl
                assert (ta // Wl) % Hl == ((t // Wl) % Hl) // s * s
    # Hl = 45, s = 4: the last group of a frame is row 44 alone
    assert oracle.anchor_index_of_token(44 * 5, 1, 45, 5, 0, 4) == 11 * 5


def test_repeat_rows_equal_their_anchor_and_stride1_is_plain(tiny_inputs):
    wl, qkv = tiny_inputs
    q, k, v = (to64(t) for t in qkv[0])
    s = wl.shape
    B = s.block
    scale = 1.0 / np.sqrt(s.D)
    nb = s.nblk
    rng = np.random.default_rng(12)
    mask = (rng.random((s.H, nb, nb)) < 0.5).astype(np.uint8)
    mask[:, :, 0] = 1
    rep = [False, True]
    O, L = oracle.sparse_attention_repeat(q, k, v, scale, B, mask, rep, s.F, s.Hl, s.Wl, 0, 2)
    # non-repeat head equals plain sparse attention
    O0, L0 = oracle.sparse_attention(q[:1], k[:1], v[:1], scale, B, mask[:1])
    np.testing.assert_array_equal(O[0], O0[0])
    # every token of the repeat head equals its anchor's row, bit for bit
    for t in range(s.N):
        a = oracle.anchor_index_of_token(t, s.F, s.Hl, s.Wl, 0, 2)
        ta = int(oracle.anchor_rows(s.F, s.Hl, s.Wl, 0, 2)[a])
        np.testing.assert_array_equal(O[1, t], O[1, ta])
    # anchor outputs = SDPA over the gathered anchor queries with the anchor-space mask
    A = oracle.anchor_rows(s.F, s.Hl, s.Wl, 0, 2)
    nqa = -(-len(A) // B)
    tm = _token_mask(mask[1, :nqa], B, len(A), s.N)
    ref = _sdpa(q[1, A][None], k[1:2], v[1:2], scale, tm[None])[0]
    np.testing.assert_allclose(O[1, A], ref, rtol=1e-11, atol=1e-12)
    # stride 1 = plain attention on every head
    O1, _ = oracle.sparse_attention_repeat(q, k, v, scale, B, mask, [True, True], s.F, s.Hl, s.Wl, 0, 1)
    Op, _ = oracle.sparse_attention(q, k, v, scale, B, mask)
    np.testing.assert_allclose(O1, Op, rtol=0, atol=0)


def test_csr_round_trip_and_schedule_order():
    rng = np.random.default_rng(13)
    H, nq, nk = 3, 7, 9
    m = (rng.random((H, nq, nk)) < 0.3).astype(np.uint8)
    m[1, 2] = 0                                     # an empty row
    rp, ci = oracle.mask_to_csr(m)
    assert rp[0] == 0 and rp[-1] == m.sum() and rp.dtype == np.int32 and ci.dtype == np.int16
    back = np.zeros_like(m)
    for r in range(H * nq):
        cols = ci[rp[r]:rp[r + 1]]
        assert np.all(np.diff(cols) > 0)
        back.reshape(H * nq, nk)[r, cols] = 1
    np.testing.assert_array_equal(back, m)
    w = oracle.build_schedule(rp, H, nq)
    rows = (w >> 16) * nq + (w & 0xFFFF)
    assert sorted(rows.tolist()) == list(range(H * nq))
    cnt = np.diff(rp)[rows]
    # heads in order; inside a head count descending, then row index ascending
    # (independent check with numpy's lexsort)
    ref = np.lexsort((np.arange(H * nq), -np.diff(rp), np.arange(H * nq) // nq))
    np.testing.assert_array_equal(rows, ref)
    for h in range(H):
        assert np.all(np.diff(cnt[h * nq:(h + 1) * nq]) <= 0)
