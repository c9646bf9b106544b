"""Seeded synthetic inputs shaped like the video-DiT attention workloads.

This module only *makes inputs*: Q/K/V tensors with a spatio-temporal
structure, static block masks drawn from a geometric recipe, and per-head
flags.  It contains none of the method's arithmetic (no softmax, no block
energies, no selection, no skip-list build): both the CUDA path and the
float64 oracle consume what it produces, and neither imports the other.

Token order for a video of F frames on an Hl x Wl latent grid is
n = (f*Hl + y)*Wl + x, followed by n_text text tokens (Mochi-style joint
attention).  Tensors are [H, N, D] (batch 1), D innermost.

Q/K/V recipe.  Each token gets a random-Fourier-feature embedding of its
scaled position p~ = (f/2, y/4, x/4):  Phi(p) = sqrt(2/r) cos(Omega p~ + beta),
Omega ~ N(0, I_3)^r, beta ~ U[0, 2pi)^r (text tokens get Phi = 0).  Per head,
U_h ~ N(0,1)^{r x D} and  X = Z_x + s * Phi U_h  (X in {Q, K, V}, Z ~ N(0,1)),
cast to bf16.  Phi(p).Phi(p') approximates a Gaussian kernel of the position
difference, so q.k carries a term ~ s^2 sqrt(D) k(p, p'): attention is local in
(f, y, x) and block energies are structured, as in the video models the
CalibAtt summaries describe (observations on sparsity and locality).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch


@dataclass(frozen=True)
class VideoShape:
    """Geometry of one attention call (batch 1)."""
    H: int            # heads
    D: int            # head dim
    F: int            # latent frames
    Hl: int           # latent rows per frame
    Wl: int           # latent columns per frame
    n_text: int = 0   # text tokens appended after the video tokens
    block: int = 128  # block size B (query and key)

    @property
    def n_video(self) -> int:
        return self.F * self.Hl * self.Wl

    @property
    def N(self) -> int:
        return self.n_video + self.n_text

    @property
    def nblk(self) -> int:
        return (self.N + self.block - 1) // self.block


@dataclass(frozen=True)
class Workload:
    """A named workload: shape plus the recipe knobs for its inputs."""
    name: str
    shape: VideoShape
    rank: int                 # rank r of the positional term
    pos_scale: float = 1.5    # s
    density: Optional[float] = None          # target block density of the seeded mask
    density_range: Optional[tuple] = None    # per-head U[lo, hi] density (mean ~ midpoint)
    repeat_heads: tuple = ()                 # heads flagged for spatial repetition
    repeat_stride: int = 1                   # anchor stride along latent rows
    timesteps: int = 1
    density_schedule: Optional[tuple] = None  # per-timestep densities
    extra: dict = field(default_factory=dict)


# The five workloads (tiny parity case, three model-shaped calls, calibration sweep).
WORKLOADS = {
    "tiny": Workload(
        "tiny", VideoShape(H=2, D=64, F=4, Hl=8, Wl=16, block=64), rank=8,
        repeat_heads=(1,), repeat_stride=2,
        extra=dict(n_calib=3, tau=0.95, rho=(1, 2))),
    "wan13b": Workload(
        "wan13b", VideoShape(H=12, D=128, F=21, Hl=30, Wl=52), rank=16, density=0.35),
    "wan14b720p": Workload(
        "wan14b720p", VideoShape(H=40, D=128, F=21, Hl=45, Wl=80), rank=16,
        density_range=(0.15, 0.45), repeat_heads=tuple(h for h in range(40) if h % 4 == 3),
        repeat_stride=4),
    "mochi1": Workload(
        "mochi1", VideoShape(H=24, D=128, F=28, Hl=30, Wl=53, n_text=256), rank=16,
        timesteps=8, density_schedule=tuple(0.50 - 0.30 * t / 7 for t in range(8))),
    "sweep": Workload(
        "sweep", VideoShape(H=12, D=128, F=21, Hl=30, Wl=52), rank=16,
        timesteps=8, extra=dict(n_calib=4, taus=(0.9, 0.95, 0.99),
                                densities=(0.10, 0.20, 0.30, 0.50, 1.00))),
}
WORKLOAD_INDEX = {"tiny": 0, "wan13b": 1, "wan14b720p": 2, "mochi1": 3, "sweep": 4}


def token_coords(shape: VideoShape):
    """(f, y, x) of every video token, plus a boolean 'is text' vector, as numpy arrays."""
    n = np.arange(shape.N)
    is_text = n >= shape.n_video
    nv = np.minimum(n, shape.n_video - 1)
    x = nv % shape.Wl
    y = (nv // shape.Wl) % shape.Hl
    f = nv // (shape.Wl * shape.Hl)
    return f, y, x, is_text


def make_qkv(wl: Workload, input_idx: int = 0, device="cpu", pos_scale: Optional[float] = None,
             dtype=torch.bfloat16, heads: Optional[int] = None, seed: Optional[int] = None):
    """Seeded Q, K, V of shape [H, N, D] in bf16 on `device`.

    The generator is torch.Generator(device) seeded 1000*cfg + input_idx (or
    seed + input_idx for ad-hoc shapes); draw order
    Omega, beta, then per head U_h, Z_q, Z_k, Z_v.  The same seed on the same device
    type gives the same tensors on every call.
    """
    shp = wl.shape
    H = shp.H if heads is None else heads
    s = wl.pos_scale if pos_scale is None else pos_scale
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed((1000 * WORKLOAD_INDEX[wl.name] if seed is None else seed) + input_idx)
    r = wl.rank
    omega = torch.randn(r, 3, generator=g, device=dev, dtype=torch.float32)
    beta = torch.rand(r, generator=g, device=dev, dtype=torch.float32) * (2 * math.pi)
    f, y, x, is_text = token_coords(shp)
    pos = torch.stack([torch.as_tensor(f, dtype=torch.float32) / 2.0,
                       torch.as_tensor(y, dtype=torch.float32) / 4.0,
                       torch.as_tensor(x, dtype=torch.float32) / 4.0], dim=1).to(dev)
    phi = math.sqrt(2.0 / r) * torch.cos(pos @ omega.T + beta)          # [N, r]
    phi[torch.as_tensor(is_text, device=dev)] = 0.0
    N, D = shp.N, shp.D
    q = torch.empty(H, N, D, dtype=dtype, device=dev)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    for h in range(H):
        u = torch.randn(r, D, generator=g, device=dev, dtype=torch.float32)
        base = s * (phi @ u)                                              # [N, D]
        for dst in (q, k, v):
            z = torch.randn(N, D, generator=g, device=dev, dtype=torch.float32)
            dst[h] = (z + base).to(dtype)
    return q, k, v


def _block_centroids(shape: VideoShape):
    """Mean frame and mean latent row of the video tokens of each block (text excluded),
    the frame range of each block, and whether the block holds a text token."""
    f, y, x, is_text = token_coords(shape)
    B, nb = shape.block, shape.nblk
    fbar = np.zeros(nb)
    ybar = np.zeros(nb)
    fmin = np.zeros(nb, dtype=np.int64)
    fmax = np.zeros(nb, dtype=np.int64)
    has_text = np.zeros(nb, dtype=bool)
    for b in range(nb):
        sl = slice(b * B, min((b + 1) * B, shape.N))
        vid = ~is_text[sl]
        has_text[b] = bool(is_text[sl].any())
        if vid.any():
            fbar[b] = f[sl][vid].mean()
            ybar[b] = y[sl][vid].mean()
            fmin[b] = f[sl][vid].min()
            fmax[b] = f[sl][vid].max()
        else:
            fbar[b], ybar[b] = fbar[b - 1], ybar[b - 1]
            fmin[b], fmax[b] = fmin[b - 1], fmax[b - 1]
    return fbar, ybar, fmin, fmax, has_text


def make_block_mask(shape: VideoShape, density: float, seed: int, n_rows: Optional[int] = None,
                    n_sinks: int = 4, text_forced: bool = False) -> np.ndarray:
    """Seeded static block mask (uint8 [n_rows, nk]) for ONE head.

    Forced set per query block i: key blocks whose frame range meets i's (frame-local
    band), key blocks within +-2 frames and one block-row extent of i's centroid
    (temporal band), `n_sinks` random sink blocks, and, when `text_forced`, every key
    block holding text and every column of a query block holding text.  The rest is
    filled by ascending |dF| + |dY|/Hl (seeded jitter breaks ties) until the row holds
    k_i = round(d*nk*(1+0.3u_i)) blocks, u_i ~ U[-1,1] re-centred to mean 0.  Rows whose
    forced set exceeds k_i keep the forced set.  density >= 1 gives the all-kept mask.
    """
    rng = np.random.default_rng(seed)
    nk = shape.nblk
    nq = nk if n_rows is None else n_rows
    if density >= 1.0:
        return np.ones((nq, nk), dtype=np.uint8)
    fbar, ybar, fmin, fmax, has_text = _block_centroids(shape)
    rows_per_block = shape.block / shape.Wl
    u = rng.uniform(-1.0, 1.0, size=nq)
    u -= u.mean()
    k_target = np.clip(np.rint(density * nk * (1.0 + 0.3 * u)).astype(np.int64), 1, nk)
    jitter = rng.uniform(0.0, 1e-3, size=(nq, nk))
    mask = np.zeros((nq, nk), dtype=np.uint8)
    qi = np.arange(nq)
    fq, yq = fbar[np.minimum(qi, nk - 1)], ybar[np.minimum(qi, nk - 1)]
    for i in range(nq):
        ii = min(i, nk - 1)
        forced = (fmin <= fmax[ii]) & (fmax >= fmin[ii])
        forced |= (np.abs(fbar - fq[i]) <= 2.0) & (np.abs(ybar - yq[i]) <= rows_per_block)
        forced[rng.choice(nk, size=min(n_sinks, nk), replace=False)] = True
        if text_forced:
            forced |= has_text
            if has_text[ii]:
                forced[:] = True
        dist = np.abs(fbar - fq[i]) + np.abs(ybar - yq[i]) / shape.Hl + jitter[i]
        dist[forced] = -1.0
        order = np.argsort(dist, kind="stable")
        kk = max(int(k_target[i]), int(forced.sum()))
        mask[i, order[:kk]] = 1
    return mask


def make_head_masks(wl: Workload, timestep: int = 0, density: Optional[float] = None,
                    seed_base: int = 0) -> np.ndarray:
    """uint8 [H, nq, nk] masks for every head of a workload (repeat heads get rows in
    anchor block space padded with zero rows up to nq).  Per-head densities follow the
    workload: a fixed value, U[lo, hi] draws, or the timestep schedule."""
    shp = wl.shape
    nq = nk = shp.nblk
    rng = np.random.default_rng(7919 * (WORKLOAD_INDEX[wl.name] + 1) + 31 * timestep + seed_base)
    if density is None:
        if wl.density_range is not None:
            dens = rng.uniform(*wl.density_range, size=shp.H)
        elif wl.density_schedule is not None:
            dens = np.full(shp.H, wl.density_schedule[timestep])
        else:
            dens = np.full(shp.H, wl.density if wl.density is not None else 0.3)
    else:
        dens = np.full(shp.H, density)
    out = np.zeros((shp.H, nq, nk), dtype=np.uint8)
    for h in range(shp.H):
        seed = int(rng.integers(0, 2**31 - 1))
        rows = nq
        if h in wl.repeat_heads:
            rows = anchor_block_count(shp, wl.repeat_stride)
        out[h, :rows] = make_block_mask(shp, float(dens[h]), seed, n_rows=rows,
                                        text_forced=shp.n_text > 0)
    return out


def anchor_block_count(shape: VideoShape, stride: int) -> int:
    """Number of query blocks in the compacted anchor sequence of a repeat head:
    F * ceil(Hl/stride) * Wl anchor tokens plus the text tokens, in blocks of B."""
    n_anchor = shape.F * (-(-shape.Hl // stride)) * shape.Wl + shape.n_text
    return (n_anchor + shape.block - 1) // shape.block


def sample_video_tokens(shape: VideoShape, n: int, seed: int = 0) -> np.ndarray:
    """n seeded video-token indices, uniform over the F*Hl*Wl video tokens (int32)."""
    rng = np.random.default_rng(seed)
    return rng.integers(0, shape.F * shape.Hl * shape.Wl, size=n).astype(np.int32)
