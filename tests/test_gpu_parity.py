"""GPU parity: every CUDA entry point against the float64 oracle on the same seeded inputs.

Bars (from the method's tolerance statement): masks, CSR lists, schedules and anchor
lists bit-exact (selection run from identical fp32 energies); block energies within
1e-4 relative (below a floor of 1e-12 * |I_i|, within 1e-16 * |I_i| absolute, since fp32
exp underflows far above fp64's range); attention outputs from bf16 inputs with fp32
accumulation within 2e-2 max-abs and 2e-3 mean-relative (mean |dO| / mean |O_ref|) of the
fp64 result.  That bar applies as stated to the fp32-output mode.  A bf16 output adds its
own rounding, up to half a bf16 ulp of the value (0.031 at |O| in [8, 16)), so bf16
outputs are held to 2e-2 + ulp_bf16(|O_ref|)/2 elementwise and the same 2e-3 mean-relative.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from calibrated_block_sparse_calib_b200 import ops, synth
from conftest import to64

pytestmark = pytest.mark.gpu

ATTN_MAXABS = 2e-2
ATTN_MEANREL = 2e-3
E_REL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    ops.lib()


def _shape(H, D, F, Hl, Wl, B, n_text=0, rank=8):
    return synth.Workload("adhoc", synth.VideoShape(H=H, D=D, F=F, Hl=Hl, Wl=Wl, n_text=n_text, block=B),
                          rank=rank)


def _inputs(wl, seed, device="cuda"):
    q, k, v = synth.make_qkv(wl, seed=seed)
    return q.to(device), k.to(device), v.to(device)


def half_ulp_bf16(x):
    """Half a bf16 ulp at |x| (8 significant bits): 2^(floor(log2 |x|) - 8)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return np.ldexp(1.0, np.floor(np.log2(ax)).astype(np.int64) - 8)


def check_attn(o_gpu, o_ref, rows=None):
    og = to64(o_gpu)
    if rows is not None:
        og, o_ref = og[:, rows], o_ref[:, rows]
    d = np.abs(og - o_ref)
    allow = ATTN_MAXABS + (half_ulp_bf16(o_ref) if o_gpu.dtype == torch.bfloat16 else 0.0)
    excess = float((d - allow).max())
    maxabs = float(d.max())
    meanrel = float(d.mean() / np.abs(o_ref).mean())
    assert excess <= 0 and meanrel <= ATTN_MEANREL, (maxabs, excess, meanrel)
    return maxabs, meanrel


def check_energy(e_gpu, e_ref, Nq, B):
    eg = to64(e_gpu)
    nq = e_ref.shape[1]
    rows = np.array([min((i + 1) * B, Nq) - i * B for i in range(nq)], float)[None, :, None]
    floor = 1e-12 * rows
    big = e_ref >= floor
    err = np.abs(eg - e_ref)
    assert np.all(err[big] <= E_REL * e_ref[big]), float((err[big] / e_ref[big]).max())
    assert np.all(err[~big] <= 1e-16 * np.broadcast_to(rows, e_ref.shape)[~big])
    return float((err[big] / e_ref[big]).max())


def _blist(mask_np, B, schedule=True):
    return ops.BlockList.from_mask(torch.from_numpy(mask_np).cuda(), B, schedule=schedule)


def _rand_mask(rng, H, nq, nk, p=0.4, diag=True):
    m = (rng.random((H, nq, nk)) < p).astype(np.uint8)
    if diag:
        for i in range(nq):
            m[:, i, min(i, nk - 1)] = 1
    return m


# ------------------------------------------------------------------------------------
# integer kernels: bit-exact
# ------------------------------------------------------------------------------------

def _energy_rows(rng, H, nq, nk):
    e = np.empty((H, nq, nk), np.float64)
    for h in range(H):
        for i in range(nq):
            kind = (h * nq + i) % 6
            if kind == 0:
                x = rng.random(nk)
            elif kind == 1:
                x = rng.exponential(size=nk) ** 4
            elif kind == 2:
                x = np.round(rng.random(nk) * 4) / 4
            elif kind == 3:
                x = np.exp(-40 * rng.random(nk))
            elif kind == 4:
                x = rng.random(nk) * 1e-39            # fp32 subnormal range
            else:
                x = np.zeros(nk)
                x[rng.integers(0, nk)] = 1.0
            e[h, i] = x
    return e.astype(np.float32)


@pytest.mark.parametrize("nk", [1, 7, 64, 256, 591, 1024])
@pytest.mark.parametrize("tau", [1e-7, 0.9, 0.95, 0.99, 1.0])
def test_select_bit_exact(nk, tau):
    rng = np.random.default_rng(nk * 31 + int(tau * 1000))
    H, nq = 2, 6
    e = _energy_rows(rng, H, nq, nk)
    e[1, 5] = 0.0                                                  # an all-zero row
    ref = oracle.select_mask(e, tau)
    got = ops.select_mask(torch.from_numpy(e).cuda(), tau).cpu().numpy()
    np.testing.assert_array_equal(got, ref)


def test_select_forced_and_count_accumulation():
    rng = np.random.default_rng(5)
    H, nq, nk = 3, 5, 100
    counts = torch.zeros(H, nq, nk, dtype=torch.int32, device="cuda")
    acc = np.zeros((H, nq, nk), np.int64)
    for d in range(3):
        e = _energy_rows(rng, H, nq, nk)
        force = (rng.random((H, nq, nk)) < 0.05).astype(np.uint8)
        ref = oracle.select_mask(e, 0.9, force_keep=force)
        got = ops.select_mask(torch.from_numpy(e).cuda(), 0.9, force_keep=torch.from_numpy(force).cuda(),
                              count_accum=counts).cpu().numpy()
        np.testing.assert_array_equal(got, ref)
        acc += ref
    np.testing.assert_array_equal(counts.cpu().numpy(), acc)


def _hard_rows(rng, H, nq, nk):
    """Rows that stress the selection kernel's two search paths: the answer's exponent level
    holding 1, ~20, ~50 (two per lane) or all of the row's blocks (equal energies), blocks of
    -0.0, and values straddling a power of two."""
    e = _energy_rows(rng, H, nq, nk).astype(np.float64)
    for h in range(H):
        for i in range(nq):
            kind = (h * nq + i) % 5
            if kind == 0:
                e[h, i] = 0.25                                     # all equal
            elif kind == 1:
                x = np.full(nk, 2.0 ** -20)
                x[rng.choice(nk, size=min(nk, 50), replace=False)] = 1.0 + rng.random(min(nk, 50)) * 0.5
                e[h, i] = x
            elif kind == 2:
                x = rng.random(nk) * 0.01
                x[rng.choice(nk, size=min(nk, 20), replace=False)] = 1.0 + rng.random(min(nk, 20))
                e[h, i] = x
            elif kind == 3:
                e[h, i] = np.where(rng.random(nk) < 0.5, 1.0, 1.0 - 2.0 ** -24)      # either side of 2^0
    e = e.astype(np.float32)
    e[0, 0, :: 3] = np.float32(-0.0)
    return e


@pytest.mark.parametrize("nk", [1, 2, 33, 64, 100, 101, 255, 256, 300, 350, 591, 600, 999, 1024])
def test_select_batched_bit_exact(nk):
    """One launch over nb entries, each at its own tau, with shared forced blocks, per-entry
    masks and vote counts: every entry's mask equals the oracle's selection of that entry,
    and the counts equal the sum of the masks.  The widths cover every energies-per-lane
    count (2, 4, 8, 16, 20, 32) with rows that are 16-byte aligned (nk % 4 == 0: vector
    loads) and rows that are not (staged through shared memory)."""
    rng = np.random.default_rng(1000 + nk)
    taus = [1e-7, 0.5, 0.9, 0.95, 0.99, 1.0]
    H, nq = 2, 5
    e = np.stack([_hard_rows(rng, H, nq, nk) for _ in taus])
    force = (rng.random((H, nq, nk)) < 0.03).astype(np.uint8)
    counts = torch.full((H, nq, nk), 7, dtype=torch.int32, device="cuda")    # counts add to what is there
    got = ops.select_mask_batched(torch.from_numpy(e).cuda(), taus, force_keep=torch.from_numpy(force).cuda(),
                                  count_accum=counts).cpu().numpy()
    acc = np.full((H, nq, nk), 7, np.int64)
    for b, tau in enumerate(taus):
        ref = oracle.select_mask(e[b], tau, force_keep=force)
        np.testing.assert_array_equal(got[b], ref, err_msg=f"entry {b} tau {tau}")
        acc += ref
    np.testing.assert_array_equal(counts.cpu().numpy(), acc)
    ops.device_check()


def _coarse_rows(rng, nrows, nk):
    """Rows of three blocks at 1.0 and tiny energies over six exponent levels, 2^-26 to 2^-35
    of the maximum.  Their integers are coarser than the float spacing, so neighbouring
    patterns share a q.  Half the tiny energies sit within 3 ulps of a half-level edge (a
    pattern with the low 22 bits 0), half are spread over the level."""
    out = np.zeros((nrows, nk), np.float32)
    for r in range(nrows):
        big = rng.choice(nk, size=3, replace=False)
        e0 = int(rng.integers(26, 30))
        lev = np.float32(2.0) ** -(e0 + rng.integers(0, 6, nk)).astype(np.float32)
        near = lev * np.array([1.0, 1.5], np.float32)[rng.integers(0, 2, nk)]
        ulp = rng.integers(-3, 4, nk).astype(np.int64)
        near = (near.view(np.int32).astype(np.int64) + ulp).astype(np.int32).view(np.float32)
        spread = (lev * (1.0 + rng.random(nk))).astype(np.float32)
        x = np.where(rng.random(nk) < 0.5, near, spread).astype(np.float32)
        x[big] = np.float32(1.0)
        out[r] = x
    return out


@pytest.mark.parametrize("nk", [100, 256, 591])
def test_select_coarse_quantisation_at_bin_edges(nk):
    """Thresholds inside the tiny energies of _coarse_rows: tau puts T a tenth, half and nine
    tenths of the way through their integer mass.  Ties between the threshold's bin and its
    neighbours are possible there, so the kernel's check at the bin's edges decides both
    ways across these rows (about a third take the exact bisection).  Each row is one batch
    entry with its own tau; every mask equals the oracle's."""
    rng = np.random.default_rng(4242 + nk)
    e, taus = [], []
    for r in _coarse_rows(rng, 40, nk):
        qi, Q = oracle.quantize_row(r)
        big = int(qi[r == np.float32(1.0)].sum())
        for f in (0.1, 0.5, 0.9):
            e.append(r)
            taus.append(min(1.0, (big + f * (Q - big)) / Q))
    e = np.stack(e)[:, None, None, :]
    got = ops.select_mask_batched(torch.from_numpy(e).cuda(), taus).cpu().numpy()
    for b, tau in enumerate(taus):
        np.testing.assert_array_equal(got[b], oracle.select_mask(e[b], tau), err_msg=f"entry {b} tau {tau}")
    ops.device_check()


def test_select_batched_many_entries_split_over_warps():
    """Enough rows x entries that each row's entries are split into chunks handled by
    different warps (vote counts then combine atomically); counts only, no masks."""
    rng = np.random.default_rng(77)
    nb, H, nq, nk = 20, 4, 250, 64
    e = np.stack([_energy_rows(rng, H, nq, nk) for _ in range(nb)])
    taus = [0.8 + 0.01 * b for b in range(nb)]
    counts = torch.zeros((H, nq, nk), dtype=torch.int32, device="cuda")
    assert ops.select_mask_batched(torch.from_numpy(e).cuda(), taus, count_accum=counts, write_masks=False) is None
    acc = sum(oracle.select_mask(e[b], taus[b]).astype(np.int64) for b in range(nb))
    np.testing.assert_array_equal(counts.cpu().numpy(), acc)
    masks = ops.select_mask_batched(torch.from_numpy(e).cuda(), taus).cpu().numpy()
    for b in (0, 7, 19):
        np.testing.assert_array_equal(masks[b], oracle.select_mask(e[b], taus[b]))


@pytest.mark.parametrize("workload,nb", [("wan13b", 32), ("wan14b720p", 2)])
def test_select_batched_full_size_sampled_rows(workload, nb):
    """The selection launch bench.py times, at full size: nb distinct energy matrices of the
    workload's shape (the GPU energy pass on its inputs, each entry rescaled per row by a
    seeded factor), tau(t) = 0.99 / 0.95 / 0.9 over the entries.  Sampled (entry, row) pairs
    are bit-exact against the oracle's selection of the same energies."""
    wl = synth.WORKLOADS[workload]
    s = wl.shape
    q, k, _ = synth.make_qkv(wl, device="cuda")
    E = ops.block_energy(q, k, s.block)
    del q, k
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    batch = torch.stack([E * (0.5 + torch.rand(E.shape[:2] + (1,), generator=g, device="cuda"))
                         for _ in range(nb)]).contiguous()
    taus = [0.99 if b < nb * 3 // 8 else (0.95 if b < nb * 6 // 8 else 0.9) for b in range(nb)]
    got = ops.select_mask_batched(batch, taus)
    ops.device_check()
    rng = np.random.default_rng(9)
    for _ in range(120):
        b, h, i = int(rng.integers(nb)), int(rng.integers(s.H)), int(rng.integers(s.nblk))
        e = batch[b, h, i].cpu().numpy()
        ref = oracle.select_row(e, taus[b], i).astype(np.uint8)
        np.testing.assert_array_equal(got[b, h, i].cpu().numpy(), ref, err_msg=f"entry {b} head {h} row {i}")


@pytest.mark.parametrize("n_inputs,rho", [(1, (1, 2)), (3, (1, 2)), (4, (1, 2)), (5, (1, 3)), (4, (0, 1))])
def test_aggregate_bit_exact(n_inputs, rho):
    rng = np.random.default_rng(n_inputs * 7 + rho[0])
    c = rng.integers(0, n_inputs + 1, size=(3, 9, 70)).astype(np.int32)
    c[1, 3] = 0
    c[1, 3, 5] = 1                                                   # a row the vote may empty
    ref = oracle.aggregate_masks(c, n_inputs, *rho)
    got = ops.aggregate_masks(torch.from_numpy(c).cuda(), n_inputs, rho).cpu().numpy()
    np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("H,nq,nk", [(1, 1, 1), (2, 8, 8), (3, 37, 53), (40, 158, 591)])
def test_csr_and_schedule_bit_exact(H, nq, nk):
    rng = np.random.default_rng(H * nq + nk)
    m = _rand_mask(rng, H, nq, nk, p=0.3, diag=False)
    if H * nq > 2:
        m[0, nq - 1] = 0                                              # an empty row
    rp_ref, ci_ref = oracle.mask_to_csr(m)
    rp, ci = ops.mask_to_csr(torch.from_numpy(m).cuda())
    rp = rp.cpu().numpy()
    np.testing.assert_array_equal(rp, rp_ref)
    np.testing.assert_array_equal(ci.cpu().numpy()[: rp[-1]], ci_ref)
    w = ops.build_schedule(torch.from_numpy(rp).cuda(), H, nq).cpu().numpy()
    np.testing.assert_array_equal(w, oracle.build_schedule(rp_ref, H, nq))


@pytest.mark.parametrize("H,nq,nk,p", [(3, 40, 70, 0.1), (2, 33, 257, 0.5), (4, 17, 1000, 0.95)])
def test_intervals_bit_exact_and_round_trip(H, nq, nk, p):
    rng = np.random.default_rng(nq * 7 + nk)
    m = _rand_mask(rng, H, nq, nk, p=p, diag=False)
    m[0, 0] = 0
    m[-1, -1] = 1
    rp, ci = oracle.mask_to_csr(m)
    ip_ref, st_ref, ln_ref = oracle.csr_to_intervals(rp, ci)
    rp_t = torch.from_numpy(rp).cuda()
    ci_t = torch.from_numpy(ci).cuda()
    ip, st, ln = ops.csr_to_intervals(rp_t, ci_t, H, nq)
    np.testing.assert_array_equal(ip.cpu().numpy(), ip_ref)
    np.testing.assert_array_equal(st.cpu().numpy(), st_ref)
    np.testing.assert_array_equal(ln.cpu().numpy(), ln_ref)
    rp2, ci2 = ops.intervals_to_csr(ip, st, ln, H, nq)
    np.testing.assert_array_equal(rp2.cpu().numpy(), rp)
    np.testing.assert_array_equal(ci2.cpu().numpy(), ci)


def test_intervals_generator_masks_and_empty_list():
    wl = synth.WORKLOADS["wan13b"]
    m = synth.make_head_masks(wl)[:3]
    H, nq, _ = m.shape
    bl = ops.BlockList.from_mask(torch.from_numpy(m).cuda(), wl.shape.block)
    ip, st, ln = ops.csr_to_intervals(bl.row_ptr, bl.col_idx, H, nq)
    ip_ref, st_ref, ln_ref = oracle.csr_to_intervals(*oracle.mask_to_csr(m))
    np.testing.assert_array_equal(ip.cpu().numpy(), ip_ref)
    np.testing.assert_array_equal(st.cpu().numpy(), st_ref)
    np.testing.assert_array_equal(ln.cpu().numpy(), ln_ref)
    # a list with no kept block at all
    z = np.zeros((2, 5, 9), np.uint8)
    rp, ci = ops.mask_to_csr(torch.from_numpy(z).cuda())
    ip, st, ln = ops.csr_to_intervals(rp, ci, 2, 5)
    assert int(ip[-1]) == 0 and st.numel() == 0
    rp2, ci2 = ops.intervals_to_csr(ip, st, ln, 2, 5)
    assert rp2.cpu().numpy().tolist() == [0] * 11 and ci2.numel() == 0


@pytest.mark.parametrize("geom", [(4, 8, 16, 0, 2), (21, 45, 80, 0, 4), (28, 30, 53, 256, 4), (3, 7, 5, 9, 3),
                                  (2, 5, 3, 0, 1)])
def test_anchor_rows_exact(geom):
    got = ops.anchor_rows(*geom).cpu().numpy()
    np.testing.assert_array_equal(got, oracle.anchor_rows(*geom))


# ------------------------------------------------------------------------------------
# block energies
# ------------------------------------------------------------------------------------

def test_energy_tiny_all_inputs(tiny_inputs):
    wl, qkv = tiny_inputs
    B, D = wl.shape.block, wl.shape.D
    scale = 1.0 / math.sqrt(D)
    for q, k, _ in qkv:
        ref = oracle.block_energy(to64(q), to64(k), scale, B)
        got = ops.block_energy(q.cuda(), k.cuda(), B)
        check_energy(got, ref, wl.shape.N, B)


@pytest.mark.parametrize("D,B,geom", [(128, 128, (5, 10, 20)), (128, 64, (3, 9, 11)), (64, 128, (2, 13, 17)),
                                      (128, 128, (3, 9, 13)), (128, 128, (1, 8, 10))])
def test_energy_ragged(D, B, geom):
    wl = _shape(2, D, *geom, B)
    q, k, _ = _inputs(wl, seed=100 + D + B)
    scale = 1.0 / math.sqrt(D)
    ref = oracle.block_energy(to64(q), to64(k), scale, B)
    got = ops.block_energy(q, k, B)
    check_energy(got, ref, wl.shape.N, B)


@pytest.mark.parametrize("geom", [(32, 64, 64, 0), (31, 64, 64, 4095)])
def test_energy_at_the_maximum_length(geom):
    """N = 131072 tokens, the longest sequence the energy pass accepts, and 131071 (a
    ragged last key block of 127 tokens): sampled query blocks against the oracle."""
    F, Hl, Wl, n_text = geom
    wl = _shape(1, 128, F, Hl, Wl, 128, n_text=n_text)
    s = wl.shape
    assert s.N in (131072, 131071)
    q, k, _ = synth.make_qkv(wl, seed=900 + n_text)
    got = ops.block_energy(q.cuda(), k.cuda(), 128).cpu()
    blocks = [0, 517, s.nblk - 1]
    ref = oracle.block_energy(to64(q), to64(k), 1.0 / math.sqrt(128), 128, q_blocks=blocks)
    g = to64(got)[:, blocks]
    rows = np.array([min((i + 1) * 128, s.N) - i * 128 for i in blocks], float)[None, :, None]
    big = ref >= 1e-12 * rows
    err = np.abs(g - ref)
    assert np.all(err[big] <= E_REL * ref[big]), float((err[big] / ref[big]).max())
    assert np.all(err[~big] <= 1e-16 * np.broadcast_to(rows, ref.shape)[~big])
    # every query row's energies sum to one softmax row
    np.testing.assert_allclose(to64(got).sum(axis=2)[0], [min((i + 1) * 128, s.N) - i * 128 for i in range(s.nblk)],
                               rtol=1e-4)


def test_energy_cached_lse_and_accumulate(tiny_inputs):
    wl, qkv = tiny_inputs
    B, D = wl.shape.block, wl.shape.D
    scale = 1.0 / math.sqrt(D)
    q, k, _ = qkv[1]
    lse = oracle.row_lse(to64(q), to64(k), scale)
    ref = oracle.block_energy(to64(q), to64(k), scale, B, lse=lse)
    lse_t = torch.from_numpy(lse.astype(np.float32)).cuda()
    got = ops.block_energy(q.cuda(), k.cuda(), B, lse=lse_t)
    check_energy(got, ref, wl.shape.N, B)


def test_energy_accumulate_and_mean_over_three_distinct_inputs(tiny_inputs):
    """The energy-mean aggregation: the accumulate flag sums three DIFFERENT inputs'
    energies, calib_energy_mean divides by the input count, and both match the oracle's
    float64 sum and mean (energy_mean) within the energy tolerance.  Selection on the GPU's
    mean energies is bit-exact against the oracle's selection on the same energies."""
    wl, qkv = tiny_inputs
    B, D, N = wl.shape.block, wl.shape.D, wl.shape.N
    scale = 1.0 / math.sqrt(D)
    refs = [oracle.block_energy(to64(q), to64(k), scale, B) for q, k, _ in qkv]
    assert len(refs) == 3 and not np.allclose(refs[0], refs[1])
    acc = None
    for d, (q, k, _) in enumerate(qkv):
        acc = ops.block_energy(q.cuda(), k.cuda(), B, out=acc, accumulate=d > 0)
        check_energy(acc, sum(refs[:d + 1]), N, B)               # each partial sum
    esum = acc.clone()
    mean = ops.energy_mean(acc, len(qkv))
    check_energy(mean, oracle.energy_mean(refs).astype(np.float64), N, B)
    # the mean is the correctly rounded fp32 quotient of the fp32 sum
    np.testing.assert_array_equal(mean.cpu().numpy(), esum.cpu().numpy() / np.float32(3))
    inplace = ops.energy_mean(esum, len(qkv), out=esum)
    assert inplace.data_ptr() == esum.data_ptr()
    np.testing.assert_array_equal(inplace.cpu().numpy(), mean.cpu().numpy())
    for tau in (0.5, 0.9, 0.95, 0.99):
        got = ops.select_mask(mean, tau).cpu().numpy()
        np.testing.assert_array_equal(got, oracle.select_mask(mean.cpu().numpy(), tau))


@pytest.mark.parametrize("count", [1, 3, 4, 1001, 4096 * 33 + 2])
def test_energy_mean_sizes(count):
    rng = np.random.default_rng(count)
    x = (rng.random(count) * 7).astype(np.float32)
    got = ops.energy_mean(torch.from_numpy(x).cuda(), 7).cpu().numpy()
    np.testing.assert_array_equal(got, x / np.float32(7))


@pytest.mark.parametrize("geom", [(2, 64, 4, 8, 16, 64), (2, 128, 6, 10, 23, 128)])
def test_energy_from_attention_lse(geom):
    """LSE reuse (the AdaSpa-style step): a dense forward emits the row LSE, and the energy
    pass takes it and runs a single pass.  The result must match the oracle's energies
    (exact fp64 LSE), which two-pass energies do as well."""
    H, D, F, Hl, Wl, B = geom
    wl = _shape(H, D, F, Hl, Wl, B)
    q, k, v = _inputs(wl, seed=41)
    N = wl.shape.N
    nb = -(-N // B)
    _, lse = ops.sparse_attn_fwd(q, k, v, _blist(np.ones((H, nb, nb), np.uint8), B), return_lse=True)
    ref = oracle.block_energy(to64(q), to64(k), 1.0 / math.sqrt(D), B)
    got = ops.block_energy(q, k, B, lse=lse)
    check_energy(got, ref, N, B)


def test_energy_anchor_rows(tiny_inputs):
    wl, qkv = tiny_inputs
    s = wl.shape
    B = s.block
    q, k, _ = qkv[0]
    rows = oracle.anchor_rows(s.F, s.Hl, s.Wl, 0, 2)
    ref = oracle.block_energy(to64(q), to64(k), 1.0 / math.sqrt(s.D), B, q_rows=rows)
    q_rows = ops.anchor_rows(s.F, s.Hl, s.Wl, 0, 2)
    got = ops.block_energy(q.cuda(), k.cuda(), B, q_rows=q_rows)
    check_energy(got, ref, len(rows), B)


# ------------------------------------------------------------------------------------
# attention
# ------------------------------------------------------------------------------------

@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_attention_tiny_random_and_dense(tiny_inputs, out_dtype):
    wl, qkv = tiny_inputs
    B, D, N = wl.shape.block, wl.shape.D, wl.shape.N
    scale = 1.0 / math.sqrt(D)
    q, k, v = qkv[0]
    rng = np.random.default_rng(1)
    nb = wl.shape.nblk
    for m in (_rand_mask(rng, 2, nb, nb, 0.4), np.ones((2, nb, nb), np.uint8)):
        O_ref, L_ref = oracle.sparse_attention(to64(q), to64(k), to64(v), scale, B, m)
        O, L = ops.sparse_attn_fwd(q.cuda(), k.cuda(), v.cuda(), _blist(m, B), return_lse=True,
                                   out_dtype=out_dtype)
        assert O.dtype == out_dtype
        check_attn(O, O_ref)
        np.testing.assert_allclose(to64(L), L_ref, rtol=0, atol=2e-4)


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("D,B,geom,p", [(128, 128, (5, 10, 20), 0.35), (128, 64, (3, 9, 11), 0.5),
                                        (64, 128, (2, 13, 17), 0.6), (128, 128, (1, 1, 70), 1.0),
                                        (128, 128, (3, 17, 40), 0.2)])
def test_attention_ragged(D, B, geom, p, out_dtype):
    wl = _shape(3, D, *geom, B)
    q, k, v = _inputs(wl, seed=200 + D + B + geom[2])
    nb = wl.shape.nblk
    m = _rand_mask(np.random.default_rng(geom[2]), 3, nb, nb, p)
    O_ref, L_ref = oracle.sparse_attention(to64(q), to64(k), to64(v), 1.0 / math.sqrt(D), B, m)
    O, L = ops.sparse_attn_fwd(q, k, v, _blist(m, B), return_lse=True, out_dtype=out_dtype)
    check_attn(O, O_ref)
    np.testing.assert_allclose(to64(L), L_ref, rtol=0, atol=2e-4)


def test_attention_empty_rows_write_zero():
    wl = _shape(2, 128, 2, 8, 30, 128)
    q, k, v = _inputs(wl, seed=300)
    nb = wl.shape.nblk
    m = _rand_mask(np.random.default_rng(3), 2, nb, nb, 0.5)
    m[0, 1] = 0
    m[1, nb - 1] = 0
    O_ref, _ = oracle.sparse_attention(to64(q), to64(k), to64(v), 1 / math.sqrt(128), 128, m)
    O, L = ops.sparse_attn_fwd(q, k, v, _blist(m, 128), return_lse=True)
    O = O.cpu()
    assert torch.all(O[0, 128:256] == 0) and torch.all(torch.isneginf(L[0, 128:256].cpu()))
    check_attn(O, O_ref)


def test_persistent_work_order_and_subsets():
    """The attention CTAs take work items by cancelling not-yet-started CTAs, so the set of
    items processed is exactly the work list, whatever its order: a random permutation of
    the schedule gives bitwise the same output (each item's arithmetic does not depend on
    the order), a list without some rows leaves those rows untouched, and repeated calls
    on the same list agree."""
    wl = _shape(3, 128, 6, 10, 23, 128)
    q, k, v = _inputs(wl, seed=77)
    nb = wl.shape.nblk
    rng = np.random.default_rng(12)
    m = _rand_mask(rng, 3, nb, nb, 0.3)
    m[1, 2] = 0                                                    # an empty row
    bl = _blist(m, 128)
    ref, lse_ref = ops.sparse_attn_fwd(q, k, v, bl, return_lse=True)
    O_ref, _ = oracle.sparse_attention(to64(q), to64(k), to64(v), 1 / math.sqrt(128), 128, m)
    check_attn(ref, O_ref)
    for trial in range(3):
        perm = torch.from_numpy(rng.permutation(bl.work.cpu().numpy()).astype(np.int32)).cuda()
        blp = ops.BlockList(bl.H, bl.nq, bl.nk, bl.block, bl.row_ptr, bl.col_idx, perm)
        o, l = ops.sparse_attn_fwd(q, k, v, blp, return_lse=True)
        assert torch.equal(o, ref) and torch.equal(l, lse_ref), trial
    # a subset of the items: the rows left out keep what the output held before
    keep = rng.random(bl.work.numel()) < 0.6
    sub = bl.work[torch.from_numpy(keep).cuda()].contiguous()
    bls = ops.BlockList(bl.H, bl.nq, bl.nk, bl.block, bl.row_ptr, bl.col_idx, sub)
    out = torch.full_like(ref, 7.0)
    ops.sparse_attn_fwd(q, k, v, bls, out=out)
    ops.device_check()
    rows = torch.zeros(3, wl.shape.N, dtype=torch.bool)
    for item in sub.cpu().tolist():
        h, i = item >> 16, item & 0xFFFF
        rows[h, i * 128:(i + 1) * 128] = True
    o, r = out.cpu(), ref.cpu()
    assert torch.equal(o[rows], r[rows])
    assert torch.all(o[~rows] == 7.0)


@pytest.mark.parametrize("n_items", [1, 147, 148, 149, 300])
def test_persistent_grid_sizes_around_the_sm_count(n_items):
    """Work lists shorter than, equal to and just above the 148 SMs (the first items run on
    their own CTAs, the rest are taken by cancellation) against the oracle."""
    wl = _shape(4, 64, 8, 16, 40, 64)                              # 5120 tokens, 80 blocks
    q, k, v = _inputs(wl, seed=n_items)
    nb = wl.shape.nblk
    rng = np.random.default_rng(n_items)
    m = _rand_mask(rng, 4, nb, nb, 0.2)
    bl = _blist(m, 64)
    work = bl.work[:n_items].contiguous()
    blw = ops.BlockList(bl.H, bl.nq, bl.nk, bl.block, bl.row_ptr, bl.col_idx, work)
    out = torch.zeros_like(q)
    ops.sparse_attn_fwd(q, k, v, blw, out=out)
    ops.device_check()
    items = work.cpu().tolist()
    heads = sorted({it >> 16 for it in items})
    O_ref, _ = oracle.sparse_attention(to64(q[heads]), to64(k[heads]), to64(v[heads]), 1 / 8.0, 64, m[heads])
    o = to64(out)
    for it in items:
        h, i = it >> 16, it & 0xFFFF
        sl = slice(i * 64, min((i + 1) * 64, wl.shape.N))
        ref_rows = O_ref[heads.index(h), sl]
        d = np.abs(o[h, sl] - ref_rows)
        assert float((d - (ATTN_MAXABS + half_ulp_bf16(ref_rows))).max()) <= 0, (h, i)


@pytest.mark.parametrize("with_lse", [False, True])
def test_masked_blocks_do_not_matter_bitwise(with_lse):
    # Rows keeping 0..4 blocks (one row empty): outputs are bit-identical across repeated
    # calls, when masked K/V blocks change, and whatever the processing order.  This also
    # guards the O-ready barrier handshake: a reader more than one phase behind a parity
    # wait would read O before the last PV products land.
    wl = _shape(2, 128, 4, 8, 24, 128)
    q, k, v = _inputs(wl, seed=400)
    nb = wl.shape.nblk
    m = _rand_mask(np.random.default_rng(4), 2, nb, nb, 0.3)
    m[:, :, 2] = 0
    bl = _blist(m, 128)
    run = lambda kk, vv, b: ops.sparse_attn_fwd(q, kk, vv, b, return_lse=with_lse)
    first = run(k, v, bl)
    O1 = first[0] if with_lse else first
    for _ in range(5):
        again = run(k, v, bl)
        assert torch.equal(O1, again[0] if with_lse else again)
    k2, v2 = k.clone(), v.clone()
    k2[:, 256:384] = torch.randn_like(k2[:, 256:384].float()).to(torch.bfloat16) * 5
    v2[:, 256:384] = torch.randn_like(v2[:, 256:384].float()).to(torch.bfloat16) * 5
    O2 = run(k2, v2, bl)
    assert torch.equal(O1, O2[0] if with_lse else O2)
    O3 = run(k, v, _blist(m, 128, schedule=False))
    assert torch.equal(O1, O3[0] if with_lse else O3)
    O_ref, _ = oracle.sparse_attention(to64(q), to64(k), to64(v), 1 / math.sqrt(128), 128, m)
    check_attn(O1, O_ref)


def test_repeat_tiny(tiny_inputs):
    wl, qkv = tiny_inputs
    s = wl.shape
    B = s.block
    q, k, v = qkv[2]
    nb = s.nblk
    rng = np.random.default_rng(6)
    m = _rand_mask(rng, 2, nb, nb, 0.5)
    nqa = synth.anchor_block_count(s, 2)
    m[1, nqa:] = 0
    rep = [False, True]
    O_ref, L_ref = oracle.sparse_attention_repeat(to64(q), to64(k), to64(v), 1 / math.sqrt(s.D), B, m, rep,
                                                  s.F, s.Hl, s.Wl, 0, 2)
    O, L = ops.sparse_attn_fwd_repeat(q.cuda(), k.cuda(), v.cuda(), _blist(m, B), rep, s.F, s.Hl, s.Wl, 0, 2,
                                      return_lse=True)
    check_attn(O, O_ref)
    np.testing.assert_allclose(to64(L), L_ref, rtol=0, atol=2e-4)
    Oc = O.cpu()
    for t in range(s.N):                       # each row of the repeat head equals its anchor's
        a = oracle.anchor_rows(s.F, s.Hl, s.Wl, 0, 2)[oracle.anchor_index_of_token(t, s.F, s.Hl, s.Wl, 0, 2)]
        assert torch.equal(Oc[1, t], Oc[1, int(a)])


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("stride", [1, 3, 4])
def test_repeat_with_text_and_ragged_groups(stride, out_dtype):
    wl = _shape(3, 128, 3, 7, 20, 128, n_text=40)
    s = wl.shape
    q, k, v = _inputs(wl, seed=500 + stride)
    nb = s.nblk
    m = _rand_mask(np.random.default_rng(stride), 3, nb, nb, 0.5)
    nqa = synth.anchor_block_count(s, stride)
    rep = [True, False, True]
    for h in (0, 2):
        m[h, nqa:] = 0
    O_ref, L_ref = oracle.sparse_attention_repeat(to64(q), to64(k), to64(v), 1 / math.sqrt(128), 128, m, rep,
                                                  s.F, s.Hl, s.Wl, s.n_text, stride)
    O, L = ops.sparse_attn_fwd_repeat(q, k, v, _blist(m, 128), rep, s.F, s.Hl, s.Wl, s.n_text, stride,
                                      return_lse=True, out_dtype=out_dtype)
    check_attn(O, O_ref)
    np.testing.assert_allclose(to64(L), L_ref, rtol=0, atol=2e-4)


# ------------------------------------------------------------------------------------
# the whole calibration + inference pipeline at the tiny workload
# ------------------------------------------------------------------------------------

def test_calibration_pipeline_tiny(tiny_inputs):
    wl, qkv = tiny_inputs
    s = wl.shape
    B = s.block
    tau = wl.extra["tau"]
    rho = wl.extra["rho"]
    scale = 1.0 / math.sqrt(s.D)
    nb = s.nblk
    counts = torch.zeros(s.H, nb, nb, dtype=torch.int32, device="cuda")
    cnt_ref = np.zeros((s.H, nb, nb), np.int64)
    energies_gpu = []
    for q, k, _ in qkv:
        e_gpu = ops.block_energy(q.cuda(), k.cuda(), B)
        e_ref = oracle.block_energy(to64(q), to64(k), scale, B)
        check_energy(e_gpu, e_ref, s.N, B)
        energies_gpu.append(e_gpu.cpu().numpy())
        # selection from identical (GPU) energies: bit-exact
        m_gpu = ops.select_mask(e_gpu, tau, count_accum=counts).cpu().numpy()
        np.testing.assert_array_equal(m_gpu, oracle.select_mask(e_gpu.cpu().numpy(), tau))
        cnt_ref += m_gpu
    np.testing.assert_array_equal(counts.cpu().numpy(), cnt_ref)
    agg = ops.aggregate_masks(counts, len(qkv), rho).cpu().numpy()
    np.testing.assert_array_equal(agg, oracle.aggregate_masks(cnt_ref, len(qkv), *rho))
    # the same vote in one batched launch over the three inputs' energies
    counts_b = torch.zeros_like(counts)
    stack = torch.from_numpy(np.stack(energies_gpu)).cuda()
    masks_b = ops.select_mask_batched(stack, [tau] * len(qkv), count_accum=counts_b).cpu().numpy()
    np.testing.assert_array_equal(counts_b.cpu().numpy(), cnt_ref)
    for d, e in enumerate(energies_gpu):
        np.testing.assert_array_equal(masks_b[d], oracle.select_mask(e, tau))
    bl = _blist(agg, B)
    q, k, v = qkv[0]
    O_ref, _ = oracle.sparse_attention(to64(q), to64(k), to64(v), scale, B, agg)
    check_attn(ops.sparse_attn_fwd(q.cuda(), k.cuda(), v.cuda(), bl), O_ref)


# ------------------------------------------------------------------------------------
# full-size Wan-1.3B-shaped call, sampled query blocks (the bench's launch configuration)
# ------------------------------------------------------------------------------------

@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_wan13b_sampled_blocks(out_dtype):
    wl = synth.WORKLOADS["wan13b"]
    s = wl.shape
    q, k, v = synth.make_qkv(wl, device="cuda")
    mask = synth.make_head_masks(wl)
    bl = _blist(mask, s.block)
    O = ops.sparse_attn_fwd(q, k, v, bl, out_dtype=out_dtype)
    torch.cuda.synchronize()
    rng = np.random.default_rng(11)
    blocks = sorted(set(rng.choice(s.nblk - 1, size=7, replace=False).tolist()) | {s.nblk - 1})
    rows = np.concatenate([np.arange(i * s.block, min((i + 1) * s.block, s.N)) for i in blocks])
    heads = [0, 5, 11]
    qh, kh, vh = (to64(t[heads]) for t in (q, k, v))
    O_ref, _ = oracle.sparse_attention(qh, kh, vh, 1 / math.sqrt(s.D), s.block, mask[heads], q_blocks=blocks)
    check_attn(O[heads], O_ref, rows=rows)


@pytest.mark.parametrize("density", [0.10, 1.0])
def test_wan13b_density_sweep_sampled_blocks(density):
    """The density sweep's launches at full size: the 10% generator mask (many short items
    per persistent CTA) and the all-kept list (this build's dense kernel), sampled query
    blocks of three heads against the oracle, with the LSE."""
    wl = synth.WORKLOADS["wan13b"]
    s = wl.shape
    q, k, v = synth.make_qkv(wl, device="cuda")
    mask = (synth.make_head_masks(wl, density=density) if density < 1
            else np.ones((s.H, s.nblk, s.nblk), np.uint8))
    O, L = ops.sparse_attn_fwd(q, k, v, _blist(mask, s.block), return_lse=True)
    ops.device_check()
    rng = np.random.default_rng(int(density * 100))
    blocks = sorted(set(rng.choice(s.nblk - 1, size=5, replace=False).tolist()) | {s.nblk - 1})
    rows = np.concatenate([np.arange(i * s.block, min((i + 1) * s.block, s.N)) for i in blocks])
    heads = [1, 7]
    qh, kh, vh = (to64(t[heads]) for t in (q, k, v))
    O_ref, L_ref = oracle.sparse_attention(qh, kh, vh, 1 / math.sqrt(s.D), s.block, mask[heads], q_blocks=blocks)
    check_attn(O[heads], O_ref, rows=rows)
    np.testing.assert_allclose(to64(L[heads])[:, rows], L_ref[:, rows], atol=5e-4, rtol=0)


def test_wait_timeout_selftest_keeps_context_usable(tiny_inputs):
    assert ops.selftest_wait_timeout(2000) == ops.CALIB_ERR_TIMEOUT
    ops.device_check()                                   # the status word was cleared
    wl, qkv = tiny_inputs
    q, k, _ = qkv[0]
    e = ops.block_energy(q.cuda(), k.cuda(), wl.shape.block)
    ops.device_check()
    assert torch.isfinite(e).all()


def _sampled_rows(rng, nblk, block, N, k=4):
    blocks = sorted(set(rng.choice(nblk - 1, size=k - 1, replace=False).tolist()) | {nblk - 1})
    return blocks, np.concatenate([np.arange(i * block, min((i + 1) * block, N)) for i in blocks])


def test_wan14b720p_repeat_heads_sampled():
    # 40 heads x 75600 tokens; heads h % 4 == 3 use spatial repetition with stride 4 along
    # latent rows (45 rows -> anchors 0, 4, ..., 44).  Checked: one plain head and one
    # repeat head on sampled query blocks, plus every row of the repeat head equal to its
    # anchor's row.
    wl = synth.WORKLOADS["wan14b720p"]
    s = wl.shape
    q, k, v = synth.make_qkv(wl, device="cuda")
    mask = synth.make_head_masks(wl)
    rep = [h in wl.repeat_heads for h in range(s.H)]
    bl = _blist(mask, s.block)
    O = ops.sparse_attn_fwd_repeat(q, k, v, bl, rep, s.F, s.Hl, s.Wl, s.n_text, wl.repeat_stride)
    torch.cuda.synchronize()
    rng = np.random.default_rng(21)
    scale = 1 / math.sqrt(s.D)
    # plain head 0
    blocks, rows = _sampled_rows(rng, s.nblk, s.block, s.N)
    qh, kh, vh = (to64(t[0:1]) for t in (q, k, v))
    O_ref, _ = oracle.sparse_attention(qh, kh, vh, scale, s.block, mask[0:1], q_blocks=blocks)
    check_attn(O[0:1], O_ref, rows=rows)
    # repeat head 3: sampled anchor blocks, compared on the anchors' own token rows
    h = 3
    A = oracle.anchor_rows(s.F, s.Hl, s.Wl, s.n_text, wl.repeat_stride)
    nqa = -(-len(A) // s.block)
    ablocks = sorted(set(rng.choice(nqa - 1, size=3, replace=False).tolist()) | {nqa - 1})
    qa = to64(q[h])[A][None]
    kh, vh = to64(k[h:h + 1]), to64(v[h:h + 1])
    Oa, _ = oracle.sparse_attention(qa, kh, vh, scale, s.block, mask[h:h + 1, :nqa], q_blocks=ablocks)
    arows = np.concatenate([np.arange(i * s.block, min((i + 1) * s.block, len(A))) for i in ablocks])
    check_attn(O[h][A][None], Oa, rows=arows)
    Oc = O[h].cpu()
    amap = np.array([oracle.anchor_index_of_token(t, s.F, s.Hl, s.Wl, s.n_text, wl.repeat_stride)
                     for t in range(0, s.N, 997)])
    for t, a in zip(range(0, s.N, 997), amap):
        assert torch.equal(Oc[t], Oc[int(A[a])])


def test_mochi1_text_tokens_sampled():
    # 24 heads x (44520 video + 256 text) tokens, timestep 7 mask (~20% density) with every
    # key block holding text and every query block holding text kept.
    wl = synth.WORKLOADS["mochi1"]
    s = wl.shape
    q, k, v = synth.make_qkv(wl, device="cuda")
    mask = synth.make_head_masks(wl, timestep=7)
    bl = _blist(mask, s.block)
    O = ops.sparse_attn_fwd(q, k, v, bl)
    torch.cuda.synchronize()
    rng = np.random.default_rng(31)
    blocks, rows = _sampled_rows(rng, s.nblk, s.block, s.N)
    heads = [0, 23]
    qh, kh, vh = (to64(t[heads]) for t in (q, k, v))
    O_ref, _ = oracle.sparse_attention(qh, kh, vh, 1 / math.sqrt(s.D), s.block, mask[heads], q_blocks=blocks)
    check_attn(O[heads], O_ref, rows=rows)


def test_mask_dictionary_build_save_load_attend(tmp_path):
    """Dictionary of 2 timesteps x 2 layers built on the device (masks -> runs), saved,
    loaded, expanded: skip lists bit-exact to the oracle's, and attention through the
    loaded list bit-identical to attention through a list built from the mask."""
    from calibrated_block_sparse_calib_b200.dictionary import MaskDictionary
    wl = _shape(2, 64, 4, 8, 16, 64)
    s = wl.shape
    q, k, v = _inputs(wl, seed=5)
    rng = np.random.default_rng(11)
    nb = s.nblk
    d = MaskDictionary(2, 2, s.H, nb, nb, s.block)
    masks = {}
    for t in range(2):
        for l in range(2):
            m = _rand_mask(rng, s.H, nb, nb, p=0.3 + 0.2 * t)
            masks[(t, l)] = m
            d.put_mask(t, l, torch.from_numpy(m).cuda(), repeat=[False, t == 1])
    path = str(tmp_path / "masks.cbsd")
    d.save(path)
    e = MaskDictionary.load(path)
    for (t, l), m in masks.items():
        bl = e.block_list(t, l)
        rp_ref, ci_ref = oracle.mask_to_csr(m)
        np.testing.assert_array_equal(bl.row_ptr.cpu().numpy(), rp_ref)
        np.testing.assert_array_equal(bl.col_idx.cpu().numpy(), ci_ref)
        np.testing.assert_array_equal(bl.work.cpu().numpy(), oracle.build_schedule(rp_ref, s.H, nb))
        assert e.repeat_heads(t, l) == (False, t == 1)
        o1 = ops.sparse_attn_fwd(q, k, v, bl)
        o2 = ops.sparse_attn_fwd(q, k, v, _blist(m, s.block))
        assert torch.equal(o1, o2)


# ------------------------------------------------------------------------------------
# spatial-repetition detection
# ------------------------------------------------------------------------------------
# Cosines are ratios of fp32 sums of N products of fp32 P values (ex2.approx, ~2^-22
# relative) accumulated in 2 x 32 chains per half-row: worst-case relative rounding of a
# sum ~ (N / 64) * 2^-24 per chain, i.e. ~1e-4 at N = 32K; held to 5e-4 absolute on cos.
COS_ABS = 5e-4


def _members(rng, shape, n):
    return rng.integers(0, shape.F * shape.Hl * shape.Wl, size=n).astype(np.int32)


@pytest.mark.parametrize("with_lse", [False, True])
def test_repeat_similarity_tiny(tiny_inputs, with_lse):
    wl, qkv = tiny_inputs
    s = wl.shape
    q, k, _ = (t.cuda() for t in qkv[0])
    rng = np.random.default_rng(3)
    mem = _members(rng, s, 150)
    scale = 1.0 / math.sqrt(s.D)
    ref = oracle.repeat_similarity(to64(q), to64(k), scale, mem, s.F, s.Hl, s.Wl, 2)
    lse = None
    if with_lse:
        lse = torch.from_numpy(oracle.row_lse(to64(q), to64(k), scale).astype(np.float32)).cuda()
    got = ops.repeat_similarity(q, k, torch.from_numpy(mem).cuda(), s.F, s.Hl, s.Wl, 2, block=s.block, lse=lse)
    np.testing.assert_allclose(to64(got), ref, atol=COS_ABS, rtol=0)
    mean_ref, flag_ref = oracle.repeat_flags(ref, mem, s.F, s.Hl, s.Wl, 2, 0.5)
    mean, flag = ops.repeat_flags(got, torch.from_numpy(mem).cuda(), s.F, s.Hl, s.Wl, 2, 0.5)
    np.testing.assert_allclose(to64(mean), mean_ref, atol=COS_ABS)
    decisive = np.abs(mean_ref - 0.5) > COS_ABS
    np.testing.assert_array_equal(flag.cpu().numpy().astype(bool)[decisive], flag_ref[decisive])


def test_repeat_similarity_repeating_head_is_flagged():
    """Head 1's member queries copy their anchors' queries: every cosine is 1 and the head is
    flagged; head 0 (independent rows) is compared with the oracle."""
    wl = _shape(2, 128, 3, 12, 20, 128)
    s = wl.shape
    q, k, _ = synth.make_qkv(wl, seed=9)
    q = q.clone()
    for t in range(s.F * s.Hl * s.Wl):
        q[1, t] = q[1, oracle.anchor_token(t, s.F, s.Hl, s.Wl, 3)]
    q, k = q.cuda(), k.cuda()
    rng = np.random.default_rng(4)
    mem = _members(rng, s, 200)
    got = ops.repeat_similarity(q, k, torch.from_numpy(mem).cuda(), s.F, s.Hl, s.Wl, 3)
    ref = oracle.repeat_similarity(to64(q), to64(k), 1.0 / math.sqrt(s.D), mem, s.F, s.Hl, s.Wl, 3)
    np.testing.assert_allclose(to64(got), ref, atol=COS_ABS, rtol=0)
    assert np.all(np.abs(to64(got)[1] - 1.0) < COS_ABS)
    mean, flag = ops.repeat_flags(got, torch.from_numpy(mem).cuda(), s.F, s.Hl, s.Wl, 3, 0.99)
    assert flag[1].item() == 1


def test_repeat_similarity_wan13b_shape_sampled():
    wl = synth.WORKLOADS["wan13b"]
    s = wl.shape
    q, k, _ = synth.make_qkv(wl, device="cuda", heads=2)
    rng = np.random.default_rng(5)
    mem = _members(rng, s, 96)
    got = ops.repeat_similarity(q, k, torch.from_numpy(mem).cuda(), s.F, s.Hl, s.Wl, 4)
    ref = oracle.repeat_similarity(to64(q), to64(k), 1.0 / math.sqrt(s.D), mem, s.F, s.Hl, s.Wl, 4)
    np.testing.assert_allclose(to64(got), ref, atol=COS_ABS, rtol=0)


def test_calibrate_slice_energy_mean_bit_exact_from_gpu_energies():
    """The calibration driver in energy-mean mode on 3 distinct inputs: its slice mask equals
    the oracle's selection on the GPU's mean energies, and those energies match the oracle's
    float64 mean within the energy tolerance."""
    from calibrated_block_sparse_calib_b200.calibrate import calibrate_slice
    wl = _shape(2, 64, 4, 8, 16, 64)
    s = wl.shape
    B, tau = s.block, 0.9
    inputs = [tuple(t.cuda() for t in synth.make_qkv(wl, seed=300 + d)[:2]) for d in range(3)]
    force = np.zeros((2, s.nblk, s.nblk), np.uint8)
    force[:, :, 0] = 1                                          # a forced key column
    mask, repeat, _ = calibrate_slice(inputs, s.F, s.Hl, s.Wl, 0, B, tau, mode="energy_mean",
                                      force_keep=torch.from_numpy(force).cuda())
    assert repeat == [False, False]
    esum = None
    for d, (q, k) in enumerate(inputs):
        esum = ops.block_energy(q, k, B, out=esum, accumulate=d > 0)
    mean = ops.energy_mean(esum, 3).cpu().numpy()
    ref_e = oracle.energy_mean([oracle.block_energy(to64(q), to64(k), 1.0 / math.sqrt(s.D), B) for q, k in inputs])
    check_energy(torch.from_numpy(mean), ref_e.astype(np.float64), s.N, B)
    np.testing.assert_array_equal(mask.cpu().numpy(), oracle.select_mask(mean, tau, force_keep=force))
    # the vote mode's slice differs in general; both are valid calibrations of the slice
    vote, _, _ = calibrate_slice(inputs, s.F, s.Hl, s.Wl, 0, B, tau, mode="vote")
    cnt = sum(oracle.select_mask(ops.block_energy(q, k, B).cpu().numpy(), tau).astype(np.int64) for q, k in inputs)
    np.testing.assert_array_equal(vote.cpu().numpy(), oracle.aggregate_masks(cnt, 3, 1, 2))


def test_calibrate_slice_with_repeat_head_bit_exact_from_gpu_energies():
    """The calibration driver end to end on 3 inputs: head 1 (member queries copy their
    anchors) is flagged and gets an anchor-space mask, head 0 a full-space one.  Replayed
    with the oracle's selection, vote and repetition decision on the same GPU energies and
    cosines, the slice mask is bit-exact."""
    from calibrated_block_sparse_calib_b200.calibrate import calibrate_slice
    wl = _shape(2, 64, 4, 8, 16, 64)
    s = wl.shape
    B, stride, tau, rho, gamma = s.block, 2, 0.9, (1, 2), 0.99
    inputs = []
    for d in range(3):
        q, k, _ = synth.make_qkv(wl, seed=100 + d)
        q = q.clone()
        for t in range(s.N):
            q[1, t] = q[1, oracle.anchor_token(t, s.F, s.Hl, s.Wl, stride)]
        inputs.append((q.cuda(), k.cuda()))
    members = torch.from_numpy(synth.sample_video_tokens(s, 120, seed=2)).cuda()
    mask, repeat, det = calibrate_slice(inputs, s.F, s.Hl, s.Wl, 0, B, tau, rho, "vote", gamma, stride, members)
    assert repeat == [False, True]
    # replay with the oracle on the GPU's energies (bit-exact selection needs identical energies)
    mem = members.cpu().numpy()
    cos = np.concatenate([to64(ops.repeat_similarity(q, k, members, s.F, s.Hl, s.Wl, stride, B))
                          for q, k in inputs], axis=1)
    mean_ref, flag_ref = oracle.repeat_flags(cos, np.tile(mem, 3), s.F, s.Hl, s.Wl, stride, gamma)
    assert flag_ref.tolist() == [False, True]
    rows = ops.anchor_rows(s.F, s.Hl, s.Wl, 0, stride)
    nb, nqa = s.nblk, -(-rows.numel() // B)
    cnt_full = np.zeros((2, nb, nb), np.int64)
    cnt_anch = np.zeros((2, nqa, nb), np.int64)
    for q, k in inputs:
        cnt_full += oracle.select_mask(ops.block_energy(q, k, B).cpu().numpy(), tau)
        cnt_anch += oracle.select_mask(ops.block_energy(q, k, B, q_rows=rows).cpu().numpy(), tau)
    ref = oracle.aggregate_masks(cnt_full, 3, *rho)
    ref_a = oracle.aggregate_masks(cnt_anch, 3, *rho)
    ref[1] = 0
    ref[1, :nqa] = ref_a[1]
    np.testing.assert_array_equal(mask.cpu().numpy(), ref)
    # the slice's masks drive the repeat-mode attention as they are
    bl = _blist(mask.cpu().numpy(), B)
    q, k = inputs[0]
    v = synth.make_qkv(wl, seed=100)[2].cuda()
    O = ops.sparse_attn_fwd_repeat(q, k, v, bl, repeat, s.F, s.Hl, s.Wl, 0, stride)
    O_ref, _ = oracle.sparse_attention_repeat(to64(q), to64(k), to64(v), 1.0 / math.sqrt(s.D), B,
                                              mask.cpu().numpy(), repeat, s.F, s.Hl, s.Wl, 0, stride)
    check_attn(O, O_ref)


# ------------------------------------------------------------------------------------
# fixtures under tests/golden/: hand-worked cases and the Tiny workload's stored oracle
# results (no oracle call at test time)
# ------------------------------------------------------------------------------------

from golden_data import hand_worked, tiny_calibration  # noqa: E402

_HW = hand_worked()


@pytest.mark.parametrize("case", _HW["select"], ids=lambda c: f"line{c['line']}")
def test_hand_worked_select_kernel(case):
    nk, i = len(case["e"]), case["diag"]
    E = np.zeros((1, i + 1, nk), np.float32)
    E[0, i] = case["e"]
    fk = None
    if case["forced"] is not None:
        f = np.zeros((1, i + 1, nk), np.uint8)
        f[0, i] = case["forced"]
        fk = torch.from_numpy(f).cuda()
    m = ops.select_mask(torch.from_numpy(E).cuda(), case["tau"], force_keep=fk).cpu().numpy()
    np.testing.assert_array_equal(m[0, i], case["keep"])


@pytest.mark.parametrize("case", _HW["vote"], ids=lambda c: f"line{c['line']}")
def test_hand_worked_vote_kernel(case):
    c = torch.from_numpy(case["counts"].astype(np.int32)[None, None]).cuda()
    np.testing.assert_array_equal(ops.aggregate_masks(c, case["n"], case["rho"]).cpu().numpy()[0, 0], case["keep"])


@pytest.mark.parametrize("case", _HW["runs"], ids=lambda c: f"line{c['line']}")
def test_hand_worked_runs_kernel(case):
    rp, ci = ops.mask_to_csr(torch.from_numpy(case["row"][None, None]).cuda())
    ip, st, ln = ops.csr_to_intervals(rp, ci, 1, 1)
    assert st.cpu().tolist() == case["starts"] and ln.cpu().tolist() == case["lens"]
    assert ip.cpu().tolist() == [0, len(case["starts"])]


@pytest.mark.parametrize("case", _HW["anchors"], ids=lambda c: f"line{c['line']}")
def test_hand_worked_anchor_rows_kernel(case):
    rows = ops.anchor_rows(case["F"], case["Hl"], case["Wl"], case["text"], case["stride"])
    assert rows.cpu().tolist() == case["rows"]


def test_tiny_golden_pipeline():
    """The Tiny workload through the kernels against the stored oracle results: energies
    in both query spaces within 1e-4 relative; selection from the stored energies, the
    vote, the skip list and the work order bit-exact; sampled attention rows (repeat head
    included) within the attention bar."""
    g = tiny_calibration()
    w = g["workload"]
    wl = synth.WORKLOADS["tiny"]
    B = w["block"]
    qkv = [synth.make_qkv(wl, input_idx=d) for d in range(w["n_inputs"])]
    rows_a = ops.anchor_rows(w["F"], w["Hl"], w["Wl"], w["n_text"], w["stride"])
    for name, sp in g["spaces"].items():
        q_rows = rows_a if name == "anchor" else None
        Nq = w["n_anchor"] if name == "anchor" else w["N"]
        counts = torch.zeros(tuple(sp["shape"]), dtype=torch.int32, device="cuda")
        for (q, k, _), e_ref, m_ref in zip(qkv, sp["energy_f32"], sp["mask_arrays"]):
            e_gpu = ops.block_energy(q.cuda(), k.cuda(), B, q_rows=q_rows)
            check_energy(e_gpu, e_ref.astype(np.float64), Nq, B)
            m = ops.select_mask(torch.from_numpy(e_ref).cuda(), w["tau"], count_accum=counts)
            np.testing.assert_array_equal(m.cpu().numpy(), m_ref)
        np.testing.assert_array_equal(counts.cpu().numpy(), sp["counts_array"])
        vote = ops.aggregate_masks(counts, w["n_inputs"], w["rho"]).cpu().numpy()
        np.testing.assert_array_equal(vote, sp["vote_array"])
    sl = g["slice"]
    bl = _blist(sl["mask_array"], B)
    nnz = sl["row_ptr"][-1]
    assert bl.row_ptr.cpu().tolist() == sl["row_ptr"]
    assert bl.col_idx[:nnz].cpu().tolist() == sl["col_idx"]
    assert bl.work.cpu().tolist() == sl["work"]
    at = g["attention"]
    q, k, v = (t.cuda() for t in qkv[at["input"]])
    for out_dtype in (torch.float32, torch.bfloat16):
        O, L = ops.sparse_attn_fwd_repeat(q, k, v, bl, w["repeat"], w["F"], w["Hl"], w["Wl"], w["n_text"],
                                          w["stride"], return_lse=True, out_dtype=out_dtype)
        check_attn(O[:, at["rows"]], at["O_array"])
        np.testing.assert_allclose(to64(L[:, at["rows"]]), at["LSE_array"], rtol=0, atol=2e-4)


# ------------------------------------------------------------------------------------
# host-buffer attention with transfers overlapped per head chunk
# ------------------------------------------------------------------------------------

@pytest.mark.parametrize("hpc,pinned,schedule", [(1, True, True), (4, True, True), (6, True, True),
                                                 (2, False, True), (2, True, False)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_host_io_attention_equals_device_call(hpc, pinned, schedule, out_dtype):
    """Chunked host <-> device copies around the same kernel: O equals the device-resident
    call bit for bit (6 heads, ragged N = 1000, chunks of 1, 4 (uneven), 6 heads, pageable
    host memory, and a list without work order, which runs as one chunk)."""
    wl = _shape(6, 128, 5, 10, 20, 128)
    q, k, v = synth.make_qkv(wl, seed=41)
    s = wl.shape
    rng = np.random.default_rng(42)
    m = _rand_mask(rng, s.H, s.nblk, s.nblk, 0.4)
    bl = _blist(m, s.block, schedule=schedule)
    lse_h = torch.empty(s.H, s.N, dtype=torch.float32, device="cuda")
    qh, kh, vh = (t.contiguous().pin_memory() if pinned else t.contiguous() for t in (q, k, v))
    st = ops.HostStaging.allocate(s.H, s.N, s.D, "cuda", out_dtype)
    st.o.fill_(float("nan"))
    o_host = ops.sparse_attn_fwd_host(qh, kh, vh, bl, staging=st, heads_per_chunk=hpc, lse=lse_h)
    torch.cuda.current_stream().synchronize()
    O_dev, L_dev = ops.sparse_attn_fwd(q.cuda(), k.cuda(), v.cuda(), bl, return_lse=True, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert o_host.dtype == out_dtype and o_host.device.type == "cpu"
    assert torch.equal(o_host, O_dev.cpu())
    assert torch.equal(lse_h.cpu(), L_dev.cpu())
    if hpc == 1 and out_dtype == torch.float32:
        O_ref, _ = oracle.sparse_attention(to64(q), to64(k), to64(v), 1 / math.sqrt(s.D), s.block, m)
        check_attn(o_host, O_ref)


def test_host_io_attention_back_to_back_calls_reuse_staging():
    """Two calls on different inputs through the same staging buffers, queued without a
    synchronisation in between: each result belongs to its own inputs."""
    wl = _shape(4, 64, 3, 9, 11, 64)
    s = wl.shape
    a = synth.make_qkv(wl, seed=5)
    b = synth.make_qkv(wl, seed=6)
    m = _rand_mask(np.random.default_rng(7), s.H, s.nblk, s.nblk, 0.5)
    bl = _blist(m, s.block)
    st = ops.HostStaging.allocate(s.H, s.N, s.D, "cuda")
    pa = [t.contiguous().pin_memory() for t in a]
    pb = [t.contiguous().pin_memory() for t in b]
    oa = ops.sparse_attn_fwd_host(*pa, bl, staging=st, heads_per_chunk=1)
    ob = ops.sparse_attn_fwd_host(*pb, bl, staging=st, heads_per_chunk=3)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(oa, ops.sparse_attn_fwd(*(t.cuda() for t in a), bl).cpu())
    assert torch.equal(ob, ops.sparse_attn_fwd(*(t.cuda() for t in b), bl).cpu())


@pytest.mark.parametrize("hpc", [1, 2, 3])
def test_host_io_repeat_attention_equals_device_call(hpc):
    """Spatial-repetition mode through host buffers (text tokens, ragged anchor groups,
    two of three heads flagged): O and LSE equal the device-resident call bit for bit."""
    wl = _shape(3, 128, 3, 7, 20, 128, n_text=40)
    s = wl.shape
    stride = 3
    q, k, v = synth.make_qkv(wl, seed=77)
    nb = s.nblk
    m = _rand_mask(np.random.default_rng(78), 3, nb, nb, 0.5)
    nqa = synth.anchor_block_count(s, stride)
    rep = [True, False, True]
    for h in (0, 2):
        m[h, nqa:] = 0
    bl = _blist(m, 128)
    geom = (rep, s.F, s.Hl, s.Wl, s.n_text, stride)
    lse_h = torch.empty(s.H, s.N, dtype=torch.float32, device="cuda")
    o_host = ops.sparse_attn_fwd_host(*(t.contiguous().pin_memory() for t in (q, k, v)), bl, heads_per_chunk=hpc,
                                      lse=lse_h, repeat=geom)
    torch.cuda.current_stream().synchronize()
    O_dev, L_dev = ops.sparse_attn_fwd_repeat(q.cuda(), k.cuda(), v.cuda(), bl, *geom, return_lse=True)
    torch.cuda.synchronize()
    assert torch.equal(o_host, O_dev.cpu())
    assert torch.equal(lse_h.cpu(), L_dev.cpu())
