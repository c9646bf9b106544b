"""Plain float64 restatement of calibrated block-sparse attention (TEST INFRASTRUCTURE).

Slow and direct on purpose: one library primitive per step (a matmul, an exp, a sum,
a sort), no blocking or fusion beyond what the definitions state.  See the package
docstring for the citation tags and for who may import this module.

Notation: heads H, tokens N, head dim D, block size B, nq/nk query/key blocks.
Block i covers rows [iB, min((i+1)B, N)) -- a ragged last block is simply shorter.
Inputs are float arrays (bf16 tensors upcast exactly); all arithmetic is float64
unless a step states otherwise.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np


# ---------------------------------------------------------------------------------
# Logits, row log-sum-exp, block energies
# ---------------------------------------------------------------------------------

def logits(q: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """S = scale * Q K^T for one head.  q [Nq, D], k [N, D] -> [Nq, N].

    The pages state the attention matrix P is post-softmax ([fr] §2.A) but give no
    scale; the reading here is the standard 1/sqrt(D), passed in by the caller."""
    return scale * (np.asarray(q, np.float64) @ np.asarray(k, np.float64).T)


def row_lse(q: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """LSE_r = log sum_c exp(S_rc), max-subtracted.  q [H, Nq, D], k [H, N, D] -> [H, Nq].

    The normaliser of the post-softmax P whose blocks are summed ([fr] §2.A, §2.B.1);
    [AdaSpa] §2 caches exactly this quantity (the LSE) to reuse it in a later search."""
    H = q.shape[0]
    out = np.empty((H, q.shape[1]), np.float64)
    for h in range(H):
        S = logits(q[h], k[h], scale)
        m = S.max(axis=1)
        out[h] = m + np.log(np.exp(S - m[:, None]).sum(axis=1))
    return out


def _block_starts(n: int, block: int) -> np.ndarray:
    return np.arange(0, n, block)


def block_energy(q: np.ndarray, k: np.ndarray, scale: float, block: int,
                 lse: Optional[np.ndarray] = None, q_rows: Optional[np.ndarray] = None,
                 q_blocks: Optional[Sequence[int]] = None) -> np.ndarray:
    """Block energies E[h, i, j] = sum_{r in I_i, c in J_j} P[r, c], P = exp(S - LSE).

    Follows [zh] §2.2A and [de] §2A.1 ("Energie" = sum of the attention scores of a
    (query block, key block) pair, blocks of B x B, e.g. 128 x 128), [pt] §2A.2 and
    [fr] §2.B.1; P is the post-softmax attention ([fr] §2.A).  It is a *sum*, not a mean
    or a max.

    q [H, Nq_all, D], k [H, N, D].  `q_rows` (token indices, compacted order) selects
    the query sequence -- the anchor rows of a spatial-repetition head; default all N
    tokens.  `lse` [H, len(rows)] is a cached LSE (as in [AdaSpa] §2); default: computed
    over all N keys.  `q_blocks` restricts the output to those query blocks (for
    sampled checks at large N); the result is then [H, len(q_blocks), nk].
    """
    H = q.shape[0]
    N = k.shape[1]
    rows = np.arange(q.shape[1]) if q_rows is None else np.asarray(q_rows)
    Nq = len(rows)
    nq = -(-Nq // block)
    blocks = list(range(nq)) if q_blocks is None else list(q_blocks)
    kstarts = _block_starts(N, block)
    out = np.zeros((H, len(blocks), len(kstarts)), np.float64)
    for h in range(H):
        for bi, i in enumerate(blocks):
            r = rows[i * block: min((i + 1) * block, Nq)]
            S = logits(q[h][r], k[h], scale)
            if lse is None:
                m = S.max(axis=1)
                l = m + np.log(np.exp(S - m[:, None]).sum(axis=1))
            else:
                l = np.asarray(lse[h], np.float64)[i * block: min((i + 1) * block, Nq)]
            P = np.exp(S - l[:, None])
            out[h, bi] = np.add.reduceat(P, kstarts, axis=1).sum(axis=0)
    return out


def energy_mean(energies: Sequence[np.ndarray]) -> np.ndarray:
    """Energy-mean aggregation: mean over calibration inputs in float64, cast to float32.

    The alternative to the pages' mask vote: average the block energies over the
    calibration inputs, then select once.  With one input it equals that input's
    energies.  The pages themselves vote on masks (see aggregate_masks)."""
    acc = np.zeros_like(np.asarray(energies[0], np.float64))
    for e in energies:
        acc += np.asarray(e, np.float64)
    return (acc / len(energies)).astype(np.float32)


# ---------------------------------------------------------------------------------
# Minimal tau-energy selection
# ---------------------------------------------------------------------------------

def ceil_log2(n: int) -> int:
    """Smallest c with 2**c >= n (n >= 1)."""
    return (int(n) - 1).bit_length()


def quantize_row(e32: np.ndarray):
    """Exact integer image of one row of float32 energies.

    Reading (the pages fix no arithmetic for the cumulative sum): scale the row by the
    power of two 2**(52 - p - ceil(log2 nk)), where e_max < 2**p, and round half-even.
    Scaling by a power of two is exact, every q_j <= 2**(52 - ceil(log2 nk)), and the
    total Q < 2**53, so Q is exact and independent of summation order.  Returns
    (q as uint64 array, Q as a Python int)."""
    e = np.asarray(e32, dtype=np.float32).astype(np.float64)
    nk = e.shape[0]
    emax = float(e.max())
    if not emax > 0.0:
        return np.zeros(nk, np.uint64), 0
    _, p = math.frexp(emax)              # emax = m * 2**p, 0.5 <= m < 1
    shift = 52 - p - ceil_log2(nk)
    q = np.rint(np.ldexp(e, shift))      # exact scaling, then round half to even
    qi = q.astype(np.uint64)
    return qi, int(sum(int(x) for x in qi))


def select_row(e32: np.ndarray, tau: float, i: int,
               forced: Optional[np.ndarray] = None) -> np.ndarray:
    """Keep set of one query block: the fewest key blocks whose cumulative energy
    reaches tau of the row's total.

    The rule is [fr] §2.B.1 (minimal number of key blocks reaching the cumulative
    threshold eps(t)); [zh] §2.2A and [de] §2A.2 state it as keeping the highest-energy
    key blocks that carry a given share of the energy.  eps(t) is called tau here and is
    a per-call argument (the timestep schedule is the caller's, [fr] §2.B.1).

    Readings: "reaches" is >= ; the threshold is T = max(1, ceil(tau (x) Q)) with one
    IEEE double multiply; candidates are taken in order (forced first, then q desc, then
    key index asc -- any order with q desc gives a minimal set, this one fixes ties);
    forced blocks count toward T; a row with Q = 0 keeps its forced blocks plus block i
    (or block 0 when i >= nk), since a query block with no key block has no softmax.
    """
    q, Q = quantize_row(e32)
    nk = q.shape[0]
    forced = np.zeros(nk, bool) if forced is None else np.asarray(forced, bool)
    keep = forced.copy()
    if Q == 0:
        keep[i if i < nk else 0] = True
        return keep
    T = max(1, math.ceil(float(np.float64(tau) * np.float64(Q))))
    order = sorted(range(nk), key=lambda j: (not forced[j], -int(q[j]), j))
    n_forced = int(forced.sum())
    cum = 0
    for rank, j in enumerate(order):
        if rank >= n_forced and cum >= T:
            break
        keep[j] = True
        cum += int(q[j])
    return keep


def select_mask(energy32: np.ndarray, tau: float,
                force_keep: Optional[np.ndarray] = None) -> np.ndarray:
    """Binary block mask uint8 [H, nq, nk] from float32 energies, one select_row per
    (head, query block) -- one mask per (timestep, layer, head) as in [zh] §2.1 and
    [de] §2A.5."""
    e = np.asarray(energy32, np.float32)
    H, nq, nk = e.shape
    out = np.zeros((H, nq, nk), np.uint8)
    for h in range(H):
        for i in range(nq):
            f = None if force_keep is None else force_keep[h, i]
            out[h, i] = select_row(e[h, i], tau, i, f)
    return out


# ---------------------------------------------------------------------------------
# Cross-input aggregation, skip lists, schedule
# ---------------------------------------------------------------------------------

def aggregate_masks(counts: np.ndarray, n_inputs: int, rho_num: int, rho_den: int) -> np.ndarray:
    """Cross-prompt vote: keep (h, i, j) iff its keep frequency is above rho.

    [zh] §2.2A, [de] §2A.3, [pt] §2A.3 and [fr] §2.B.2: average the per-prompt binary
    masks and keep blocks whose frequency exceeds the agreement threshold rho
    (e.g. 0.5).  "Above" is strict; evaluated in integers as
    count * rho_den > rho_num * n_inputs.  Reading: a row the vote leaves empty keeps
    its most frequent key block (lowest index on ties), so every query block attends
    to something."""
    c = np.asarray(counts, np.int64)
    keep = c * int(rho_den) > int(rho_num) * int(n_inputs)
    H, nq, nk = c.shape
    for h in range(H):
        for i in range(nq):
            if not keep[h, i].any():
                keep[h, i, int(np.argmax(c[h, i]))] = True
    return keep.astype(np.uint8)


def mask_to_csr(mask: np.ndarray):
    """Skip list of a mask: per (h, i) row the ascending kept key-block indices.

    The pages turn each mask into a list holding only the block intervals to compute
    ([zh] §2.2B, [pt] §2A.5, [fr] §2.C).  Layout: row r = h*nq + i; row_ptr int32
    [H*nq + 1], col_idx int16 [nnz]."""
    m = np.asarray(mask).astype(bool)
    H, nq, nk = m.shape
    flat = m.reshape(H * nq, nk)
    counts = flat.sum(axis=1)
    row_ptr = np.zeros(H * nq + 1, np.int64)
    row_ptr[1:] = np.cumsum(counts)
    cols = [np.nonzero(flat[r])[0] for r in range(H * nq)]
    col_idx = np.concatenate(cols) if cols else np.zeros(0, np.int64)
    return row_ptr.astype(np.int32), col_idx.astype(np.int16)


def csr_to_intervals(row_ptr: np.ndarray, col_idx: np.ndarray):
    """Interval form of a skip list: per row, the maximal runs of consecutive kept key
    blocks as (start, length), in ascending order.

    The pages describe the per-query-block list as the block intervals to compute ([zh]
    §2.2B, [fr] §2.C).  Layout: iv_ptr int32 [rows + 1], starts int16, lengths int16."""
    rp = np.asarray(row_ptr, np.int64)
    ci = np.asarray(col_idx, np.int64)
    iv_ptr, starts, lens = [0], [], []
    for r in range(len(rp) - 1):
        cols = ci[rp[r]:rp[r + 1]]
        p = 0
        while p < len(cols):
            q = p + 1
            while q < len(cols) and cols[q] == cols[q - 1] + 1:
                q += 1
            starts.append(cols[p])
            lens.append(q - p)
            p = q
        iv_ptr.append(len(starts))
    return (np.array(iv_ptr, np.int32), np.array(starts, np.int16), np.array(lens, np.int16))


def intervals_to_csr(iv_ptr: np.ndarray, starts: np.ndarray, lens: np.ndarray):
    """Inverse of csr_to_intervals: every run expanded into its block indices."""
    ip = np.asarray(iv_ptr, np.int64)
    row_ptr, cols = [0], []
    for r in range(len(ip) - 1):
        for k in range(ip[r], ip[r + 1]):
            cols.extend(range(int(starts[k]), int(starts[k]) + int(lens[k])))
        row_ptr.append(len(cols))
    return np.array(row_ptr, np.int32), np.array(cols, np.int16)


def build_schedule(row_ptr: np.ndarray, H: int, nq: int) -> np.ndarray:
    """Work list for load balancing by kept-block count: heads in ascending order and,
    within a head, query blocks by kept count descending (ties by query block
    ascending); entry = h << 16 | i.

    [AdaSpa] §2 motivates balancing the kernel's load across heads of different
    sparsity; longest-first order is the classic greedy for that.  Reading: the order is
    head-major so that the key/value blocks the concurrently running tiles read belong to
    one or two heads at a time (a locality choice; the pages fix no order)."""
    rp = np.asarray(row_ptr, np.int64)
    cnt = rp[1:] - rp[:-1]
    order = sorted(range(H * nq), key=lambda r: (r // nq, -int(cnt[r]), r))
    return np.array([((r // nq) << 16) | (r % nq) for r in order], np.int32)


# ---------------------------------------------------------------------------------
# Spatial repetition: anchor rows
# ---------------------------------------------------------------------------------

def anchor_rows(F: int, Hl: int, Wl: int, n_text: int, stride: int) -> np.ndarray:
    """Token indices of the anchor rows of a spatial-repetition head, compacted order.

    [zh] §2.1/§2.2B, [de] §2A.4, [fr] §2.A.4 and §2.C: in flagged heads, rows of one
    frame share their attention pattern, so only a few anchor rows are computed and the
    result is broadcast to the other rows of the same frame.  Reading: the anchors are
    latent rows y = 0, s, 2s, ... of every frame (stride s along latent rows), every
    column x; text tokens follow and are never repeated."""
    Ar = -(-Hl // stride)
    out = []
    for f in range(F):
        for ya in range(Ar):
            y = ya * stride
            for x in range(Wl):
                out.append((f * Hl + y) * Wl + x)
    nv = F * Hl * Wl
    out.extend(range(nv, nv + n_text))
    return np.array(out, np.int64)


def anchor_index_of_token(t: int, F: int, Hl: int, Wl: int, n_text: int, stride: int) -> int:
    """Compacted anchor index whose output token t receives: token (f, y, x) takes the
    anchor (f, floor(y/s)*s, x); a text token takes its own row."""
    nv = F * Hl * Wl
    Ar = -(-Hl // stride)
    if t >= nv:
        return F * Ar * Wl + (t - nv)
    x = t % Wl
    y = (t // Wl) % Hl
    f = t // (Wl * Hl)
    return (f * Ar + y // stride) * Wl + x


def anchor_token(t: int, F: int, Hl: int, Wl: int, stride: int) -> int:
    """Token whose attention row video token t = (f, y, x) takes at stride s: the anchor
    (f, floor(y/s)*s, x).  Text tokens (t >= F*Hl*Wl) are their own anchor."""
    nv = F * Hl * Wl
    if t >= nv:
        return t
    x = t % Wl
    y = (t // Wl) % Hl
    f = t // (Wl * Hl)
    return (f * Hl + (y // stride) * stride) * Wl + x


def repeat_similarity(q: np.ndarray, k: np.ndarray, scale: float, members, F: int, Hl: int, Wl: int,
                      stride: int) -> np.ndarray:
    """cos(P[a(b)], P[b]) for every sampled token b and head h: [H, n].

    [zh] §2.2A: the cosine similarity between the attention vectors of different spatial
    rows of one frame is measured; a head whose similarity exceeds gamma is marked spatially
    repetitive ([fr] §2.B.3 likewise).  Reading: a token's attention vector is its
    post-softmax row P over all keys, and each sampled token b = (f, y, x) is compared with
    the anchor a(b) = (f, floor(y/s)*s, x) whose output it would receive."""
    H = q.shape[0]
    members = [int(b) for b in members]
    anchors = [anchor_token(b, F, Hl, Wl, stride) for b in members]
    out = np.empty((H, len(members)), np.float64)
    for h in range(H):
        rows = sorted(set(members) | set(anchors))
        idx = {r: n for n, r in enumerate(rows)}
        S = logits(q[h][rows], k[h], scale)
        P = np.exp(S - S.max(axis=1, keepdims=True))
        P /= P.sum(axis=1, keepdims=True)
        for i, (a, b) in enumerate(zip(anchors, members)):
            pa, pb = P[idx[a]], P[idx[b]]
            out[h, i] = float(pa @ pb) / np.sqrt(float(pa @ pa) * float(pb @ pb))
    return out


def repeat_flags(sim: np.ndarray, members, F: int, Hl: int, Wl: int, stride: int, gamma: float):
    """Per head: the mean similarity over the sampled tokens that are not their own anchor,
    and the flag mean > gamma ("exceeds the threshold", [zh] §2.2A).  A head with no such
    token is not flagged (mean 0)."""
    use = np.array([anchor_token(int(b), F, Hl, Wl, stride) != int(b) for b in members], bool)
    sim = np.asarray(sim, np.float64)
    mean = sim[:, use].mean(axis=1) if use.any() else np.zeros(sim.shape[0])
    return mean, mean > gamma


# ---------------------------------------------------------------------------------
# Block-sparse attention
# ---------------------------------------------------------------------------------

def sparse_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float, block: int,
                     mask: np.ndarray, q_blocks: Optional[Sequence[int]] = None,
                     heads: Optional[Sequence[int]] = None):
    """O_r = sum_{c in K(i)} softmax_{c in K(i)}(S_rc) v_c, K(i) = union of the kept key
    blocks of r's query block i; LSE_r = log sum_{c in K(i)} exp(S_rc).

    [zh] §2.2B, [de] §2B, [pt] §2B, [fr] §2.C: the kernel computes only the kept
    blocks, densely inside each.  Written as dense attention with masked logits set to
    -inf, so the all-kept mask is the dense result itself.  Reading: a query block with
    no kept key block outputs O = 0 and LSE = -inf.

    q [H, Nq, D] (its own row sequence; blocks of B over Nq), k/v [H, N, D],
    mask [H, >=nq, nk].  Rows outside `q_blocks` and heads outside `heads` are NaN.
    Returns (O [H, Nq, D], LSE [H, Nq]) in float64."""
    H, Nq, D = q.shape
    N = k.shape[1]
    nq = -(-Nq // block)
    O = np.full((H, Nq, D), np.nan)
    L = np.full((H, Nq), np.nan)
    blocks = range(nq) if q_blocks is None else q_blocks
    hs = range(H) if heads is None else heads
    for h in hs:
        kh = np.asarray(k[h], np.float64)
        vh = np.asarray(v[h], np.float64)
        for i in blocks:
            r0, r1 = i * block, min((i + 1) * block, Nq)
            allowed = np.zeros(N, bool)
            for j in np.nonzero(mask[h, i])[0]:
                allowed[j * block: min((j + 1) * block, N)] = True
            if not allowed.any():
                O[h, r0:r1] = 0.0
                L[h, r0:r1] = -np.inf
                continue
            S = logits(q[h, r0:r1], kh, scale)
            S[:, ~allowed] = -np.inf
            m = S.max(axis=1)
            W = np.exp(S - m[:, None])
            lsum = W.sum(axis=1)
            O[h, r0:r1] = (W @ vh) / lsum[:, None]
            L[h, r0:r1] = m + np.log(lsum)
    return O, L


def sparse_attention_repeat(q, k, v, scale: float, block: int, mask: np.ndarray,
                            head_repeat: Sequence[bool], F: int, Hl: int, Wl: int,
                            n_text: int, stride: int, q_blocks=None, heads=None):
    """Block-sparse attention with spatial repetition on the flagged heads.

    Unflagged heads: sparse_attention over all N query rows.  Flagged heads
    ([zh] §2.2B, [fr] §2.C): attention is computed for the anchor rows only -- the
    compacted anchor sequence, whose query blocks index the mask (anchor block space)
    -- and each token's output and LSE are its anchor's.  `q_blocks` selects query
    blocks in each head's own block space.  Returns (O [H, N, D], LSE [H, N])."""
    H, N, D = q.shape
    O = np.full((H, N, D), np.nan)
    L = np.full((H, N), np.nan)
    hs = range(H) if heads is None else heads
    A = anchor_rows(F, Hl, Wl, n_text, stride)
    amap = np.array([anchor_index_of_token(t, F, Hl, Wl, n_text, stride) for t in range(N)])
    for h in hs:
        if not head_repeat[h]:
            Oh, Lh = sparse_attention(q[h:h + 1], k[h:h + 1], v[h:h + 1], scale, block,
                                      mask[h:h + 1], q_blocks=q_blocks)
            O[h], L[h] = Oh[0], Lh[0]
            continue
        qa = np.asarray(q[h], np.float64)[A][None]
        nqa = -(-len(A) // block)
        qb = None if q_blocks is None else [i for i in q_blocks if i < nqa]
        Oa, La = sparse_attention(qa, k[h:h + 1], v[h:h + 1], scale, block,
                                  mask[h:h + 1, :nqa], q_blocks=qb)
        O[h] = Oa[0][amap]
        L[h] = La[0][amap]
    return O, L
