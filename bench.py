"""Benchmark of calibrated block-sparse attention on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload wan13b] [--impl reference]

A step is one inference call of the hot path: sparse_attn_fwd over the workload's
calibrated skip list (masks, skip lists and the longest-first schedule are built before
inference and held in memory, as the method prescribes).  Inputs are resident in HBM when
the timed region starts; Q/K/V/O of the default workload (Wan-1.3B shape: 12 heads x
32760 tokens x 128) total 403 MB, larger than L2, so no flush is needed between steps.
value = kept-only TFLOPS = 4 D sum_kept |I_i||J_j| / time, summed over ranks (each rank
runs a replica: scaling "weak").  The same line carries the dense-equivalent TFLOPS, the
roofline of the attention kernel against the measured bf16 peak, the speedup over this
build's own kernel with an all-kept list, an end-to-end figure with host<->device copies
in the timed region, the calibration pass (fused LSE + block energies, selection)
measured on the same shapes, and the float64 oracle timed on a bounded sample on the
host cores.  `--impl reference` times that oracle alone as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse attn TFLOPS (kept-only & dense-equiv) + % BF16 TC peak at 30% density"
UNIT = "TFLOPS"

# DRAM bytes (read + write) of one attn_fwd_kernel launch on the wan13b workload, from an
# ncu capture of that launch (dram__bytes_read.sum + dram__bytes_write.sum), valid only for
# the kernel sources it was taken on: reported as roofline.traffic while the source hashes
# still match, else null.
NCU_TRAFFIC = {("wan13b", "4d3844dc7507", "c7c3253ba1c1"): 302_891_520 + 86_448_896}

# MUFU exp2 throughput of one SM: 4 lanes per clock in each of the 4 sub-partitions.
MUFU_EX2_PER_CLK_SM = 16
B200_SMS = 148


def _src_sha(name):
    path = os.path.join(ROOT, "calibrated_block_sparse_calib_b200", "csrc", name)
    with open(path, "rb") as f:
        return hashlib.sha1(f.read()).hexdigest()[:12]


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return {"bf16_tflops": d["bf16_tflops"], "bf16_tflops_sustained": d["bf16_tflops_sustained"],
                "hbm_gbs": d["hbm_gbs"], "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


def max_over_ranks(x: float, dist, device) -> float:
    """The largest value of x over all ranks (every rank gets it): a multi-GPU step time is the
    slowest rank's device time."""
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput of `world` replicas that each did `flops_per_rank` in at most ms_max."""
    return flops_per_rank * world / (ms_max * 1e-3) / 1e12


def kept_flops(mask: np.ndarray, N: int, D: int, B: int, repeat_heads=(), n_anchor=None) -> float:
    """4 D sum over kept (i, j) of |I_i| |J_j| with real (ragged) block sizes; repeat heads
    count their anchor-space rows."""
    H, nq, nk = mask.shape
    kc = np.array([min((j + 1) * B, N) - j * B for j in range(nk)], np.float64)
    total = 0.0
    for h in range(H):
        Nq = n_anchor if (h in repeat_heads and n_anchor is not None) else N
        nqh = (Nq + B - 1) // B
        rows = np.array([min((i + 1) * B, Nq) - i * B for i in range(nqh)], np.float64)
        total += float(rows @ (mask[h, :nqh].astype(np.float64) @ kc))
    return 4.0 * D * total


def workload_config(wl, mask_np, n_gpus: int, n_anchor) -> dict:
    """The line's `config`, the same in both arms: the workload's shape, its kept fraction of
    the dense FLOPs (repeat heads counted by their n_anchor anchor rows), and how the inputs
    relate to L2."""
    s = wl.shape
    H, N, D, B = s.H, s.N, s.D, s.block
    rep = tuple(h for h in range(H) if h in wl.repeat_heads)
    density = kept_flops(mask_np, N, D, B, rep, n_anchor) / (4.0 * N * N * D * H)
    qkvo_mb = 4 * H * N * D * 2 / 1e6
    return {"workload": wl.name, "H": H, "N": N, "D": D, "block": B, "density": round(density, 4),
            "repeat_heads": len(rep), "parallelism": f"replicas{n_gpus}",
            "l2": f"inputs larger than L2 (Q/K/V/O {qkvo_mb:.0f} MB), no flush"}


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", self.gpu_id], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for l in getattr(self, "lines", []):
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def _time_calls(fn, steps, warmup, torch):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        fn()
    e1.record(st)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def _time_graph(fn, calls, torch, replays=5):
    """Device time per call of a short kernel: `calls` calls captured in one CUDA graph,
    replayed (after one untimed replay) between events, so that the host's per-call cost
    is not what gets measured."""
    fn()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for _ in range(calls):
                fn()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(replays):
        g.replay()
    e1.record(st)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (replays * calls)
    del g
    return ms


def _time_flushed(fn, iters, torch, flush):
    """Median device time of fn() over `iters` launches, each after a write of `flush` (a
    buffer larger than L2), so every launch reads its inputs from HBM."""
    st = torch.cuda.current_stream()
    fn()
    ts = []
    for _ in range(iters):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        fn()
        e1.record(st)
        e1.synchronize()
        ts.append(e0.elapsed_time(e1))
    return statistics.median(ts)


def select_leg(energy, taus, torch, ops, flush, peaks, iters=10):
    """One batched selection launch over energy [nb, H, nq, nk] (per-entry masks written),
    timed with L2 flushed before each launch.  Bytes: energies read + masks written."""
    nb = energy.shape[0]
    msk = torch.empty(energy.shape, dtype=torch.uint8, device=energy.device)
    ms = _time_flushed(lambda: ops.select_mask_batched(energy, taus, out=msk), iters, torch, flush)
    nbytes = energy.numel() * (4 + 1)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"shape": list(energy.shape), "entries": nb, "ms": ms, "bytes": nbytes, "gbs": gbs,
            "frac_hbm": gbs / peaks["hbm_gbs"], "kept_density": float(msk.float().mean().item()),
            "kernel": f"select_mask_kernel<{_mpl(energy.shape[-1])}>"}


def _mpl(nk):
    for m, cap in ((2, 64), (4, 128), (8, 256), (16, 512), (20, 640)):
        if nk <= cap:
            return m
    return 32


def config_leg(name, wl, timestep, dev, torch, ops, synth, peaks, steps=20, dense_iters=3, flush=None,
               with_select=False):
    """Attention on one more workload shape, each number with its own clock record: kept-only
    and dense-equivalent TFLOPS, fraction of the bf16 peak, and the speedup over this build's
    dense kernel; optionally the selection pass on that workload's energies."""
    s = wl.shape
    B, D, N, H = s.block, s.D, s.N, s.H
    q, k, v = synth.make_qkv(wl, device=dev)
    mask_np = synth.make_head_masks(wl, timestep=timestep)
    bl = ops.BlockList.from_mask(torch.from_numpy(mask_np).to(dev), B)
    rep = [h in wl.repeat_heads for h in range(H)]
    stride = wl.repeat_stride
    n_anchor = ops.anchor_count(s.F, s.Hl, s.Wl, s.n_text, stride) if any(rep) else None
    out = torch.empty_like(q)
    if any(rep):
        call = lambda: ops.sparse_attn_fwd_repeat(q, k, v, bl, rep, s.F, s.Hl, s.Wl, s.n_text, stride, out=out)
    else:
        call = lambda: ops.sparse_attn_fwd(q, k, v, bl, out=out)
    fk = kept_flops(mask_np, N, D, B, tuple(h for h in range(H) if rep[h]), n_anchor)
    fd = 4.0 * N * N * D * H
    gpu_id = _gpu_id(torch, dev)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    with ClockSampler(gpu_id) as clk:
        ms = _time_calls(call, steps, 0, torch)
    ops.device_check()
    res = {"workload": name, "H": H, "N": N, "D": D, "block": B, "timestep": timestep, "repeat_heads": sum(rep),
           "kept_fraction_of_dense": round(fk / fd, 4), "ms": ms, "kept_tflops": fk / (ms * 1e-3) / 1e12,
           "dense_equiv_tflops": fd / (ms * 1e-3) / 1e12,
           "frac_of_bf16_peak": fk / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
           "frac_of_sustained": fk / (ms * 1e-3) / 1e12 / peaks["bf16_tflops_sustained"], "clocks": clk.summary()}
    c = res["clocks"]
    if c.get("sm_mhz") and c.get("sm_max_mhz"):
        res["kept_tflops_at_max_clock"] = res["kept_tflops"] * c["sm_max_mhz"] / c["sm_mhz"]
    if dense_iters:
        full = torch.ones((H, s.nblk, s.nblk), dtype=torch.uint8, device=dev)
        bl_dense = ops.BlockList.from_mask(full, B)
        ms_dense = _time_calls(lambda: ops.sparse_attn_fwd(q, k, v, bl_dense, out=out), dense_iters, 1, torch)
        res["dense_kernel"] = {"ms": ms_dense, "tflops": fd / (ms_dense * 1e-3) / 1e12}
        res["speedup_vs_dense"] = ms_dense / ms
        del bl_dense, full
    if with_select:
        E = ops.block_energy(q, k, B)
        res["select"] = select_leg(E.unsqueeze(0), [0.95], torch, ops, flush, peaks)
        del E
    ops.device_check()
    del q, k, v, out
    torch.cuda.empty_cache()
    return res


def _gpu_id(torch, dev):
    gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
    return gpu_uuid if gpu_uuid.startswith("GPU-") else f"GPU-{gpu_uuid}"


def cpu_baseline(wl, q, k, v, mask, budget_s: float = 12.0):
    """The float64 oracle on a bounded sample: whole query blocks of head 0 (kept keys only
    enter the softmax), as many as fit in ~budget_s.  Returns kept-only TFLOPS."""
    import oracle
    from threadpoolctl import threadpool_info
    s = wl.shape
    B, D, N = s.block, s.D, s.N
    scale = 1.0 / math.sqrt(D)
    q0 = q[0:1].float().cpu().numpy().astype(np.float64)
    k0 = k[0:1].float().cpu().numpy().astype(np.float64)
    v0 = v[0:1].float().cpu().numpy().astype(np.float64)
    kc = np.array([min((j + 1) * B, N) - j * B for j in range(s.nblk)], np.float64)
    done, flops, t0 = 0, 0.0, time.perf_counter()
    while time.perf_counter() - t0 < budget_s and done < s.nblk:
        i = (done * 37) % s.nblk
        oracle.sparse_attention(q0, k0, v0, scale, B, mask[0:1], q_blocks=[i])
        rows = min((i + 1) * B, N) - i * B
        flops += 4.0 * D * rows * float(mask[0, i].astype(np.float64) @ kc)
        done += 1
    dt = time.perf_counter() - t0
    threads = max([t.get("num_threads", 1) for t in threadpool_info()] or [1])
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": int(threads), "kind": "oracle",
            "sample": f"{done} query blocks of head 0 at {wl.name} (N={N}, D={D}), {dt:.1f} s, "
                      f"float64 NumPy on {os.cpu_count()} host cores"}


def run_reference(args):
    """Reference arm: the float64 oracle, as it stands, on the host cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch
    from calibrated_block_sparse_calib_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    q, k, v = synth.make_qkv(wl, heads=1)
    full_mask = synth.make_head_masks(wl, timestep=args.timestep)
    mask = full_mask[:1]
    n_anchor = None
    if wl.repeat_heads:
        import oracle
        s = wl.shape
        n_anchor = len(oracle.anchor_rows(s.F, s.Hl, s.Wl, s.n_text, wl.repeat_stride))
    per_step = []
    for _ in range(args.warmup):
        cpu_baseline(wl, q, k, v, mask, budget_s=0.5)
    for _ in range(args.steps):
        per_step.append(cpu_baseline(wl, q, k, v, mask, budget_s=max(0.5, args.ref_seconds / max(1, args.steps))))
    val = statistics.mean(p["value"] for p in per_step)
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, full_mask, args.gpus, n_anchor),
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": per_step[0]["cores"], "kind": "oracle",
                             "sample": per_step[0]["sample"]},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_energy_only(args, wl, dev, torch, ops, synth):
    """The calibration leg alone: fused row-LSE + block-energy pass (two passes over K), then
    the selection on those energies: first one batched launch over 32 copies (the sweep's
    4 inputs x 8 timesteps, L2 flushed before each launch; the first selection launches of
    the process), then one matrix per call."""
    s = wl.shape
    H = args.heads or s.H
    q, k, _ = synth.make_qkv(wl, device=dev, heads=H)
    E = ops.block_energy(q, k, s.block)
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev)
    batch = E.unsqueeze(0).repeat(32, 1, 1, 1)
    sel_batched = select_leg(batch, [0.99 if t < 3 else (0.95 if t < 6 else 0.9) for t in range(8) for _ in range(4)],
                             torch, ops, flush, _peaks())
    del batch, flush
    ms = _time_calls(lambda: ops.block_energy(q, k, s.block, out=E), args.steps, args.warmup, torch)
    # the selection pass on these energies, with vote-count accumulation (device time)
    msk = torch.empty(E.shape, dtype=torch.uint8, device=dev)
    cnt = torch.zeros(E.shape, dtype=torch.int32, device=dev)
    ms_sel = _time_graph(lambda: ops.select_mask(E, 0.95, out=msk, count_accum=cnt), 20, torch)
    ops.device_check()
    exps = 2.0 * s.N * s.N * H / (ms * 1e-3)
    peak = MUFU_EX2_PER_CLK_SM * B200_SMS * 1965.0e6
    sel_bytes = E.numel() * (4 + 1 + 4 + 4)       # energies in, mask out, counts read + written
    hbm = _peaks()["hbm_gbs"]
    print(json.dumps({"leg": "block_energy", "workload": wl.name, "H": H, "N": s.N, "D": s.D, "block": s.block,
                      "ms": ms, "exp2_per_s": exps, "frac_of_mufu_at_1965mhz": exps / peak,
                      "select": {"shape": list(E.shape), "tau": 0.95, "ms": ms_sel,
                                 "gbs": sel_bytes / (ms_sel * 1e-3) / 1e9,
                                 "frac_hbm": sel_bytes / (ms_sel * 1e-3) / 1e9 / hbm,
                                 "kept_density": float(msk.float().mean().item())},
                      "select_batched_32": sel_batched}), flush=True)


def run_calibration_sweep(dev, torch, ops, synth):
    """Offline calibration over the sweep workload (12 heads x 32760 tokens, B=128): for each of
    8 timesteps (positional scale 1 + t/8) and 4 seeded inputs, the fused LSE + energy pass, then
    the minimal tau-selection for tau in {0.9, 0.95, 0.99} in two aggregation modes -- per-input
    masks with the cross-input vote (rho = 1/2; one batched launch over a timestep's 4 inputs
    accumulates the vote counts), and one selection on the energies averaged over the inputs
    (the kernel's accumulate flag, then the energy mean).  One more batched launch selects all
    32 (input, timestep) entries at tau(t).  Reports times, rates and the kept densities."""
    wl = synth.WORKLOADS["sweep"]
    s = wl.shape
    B, N, H, nb = s.block, s.N, s.H, s.nblk
    n_in, taus, T = wl.extra["n_calib"], wl.extra["taus"], wl.timesteps
    st = torch.cuda.current_stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)
    peaks = _peaks()
    E_all = torch.empty((T * n_in, H, nb, nb), dtype=torch.float32, device=dev)
    Esum = torch.empty((H, nb, nb), dtype=torch.float32, device=dev)
    msk = torch.empty((H, nb, nb), dtype=torch.uint8, device=dev)
    counts = torch.empty((H, nb, nb), dtype=torch.int32, device=dev)
    dens = {"vote": {str(t_): [] for t_ in taus}, "energy_mean": {str(t_): [] for t_ in taus}}
    e_ms, a_ms, sel_ms = [], [], []
    t_start = time.perf_counter()
    for t in range(T):
        qk = [synth.make_qkv(wl, input_idx=d, device=dev, pos_scale=1.0 + 0.125 * t)[:2] for d in range(n_in)]
        ops.block_energy(qk[0][0], qk[0][1], B, out=Esum)        # warm-up
        for d, (q, k) in enumerate(qk):
            e0, e1 = ev(), ev()
            e0.record(st)
            ops.block_energy(q, k, B, out=E_all[t * n_in + d])
            e1.record(st)
            torch.cuda.synchronize()
            e_ms.append(e0.elapsed_time(e1))
        for d, (q, k) in enumerate(qk):
            e0, e1 = ev(), ev()
            e0.record(st)
            ops.block_energy(q, k, B, out=Esum, accumulate=d > 0)
            e1.record(st)
            torch.cuda.synchronize()
            a_ms.append(e0.elapsed_time(e1))
        ops.energy_mean(Esum, n_in, out=Esum)
        for tau in taus:
            dens["energy_mean"][str(tau)].append(float(ops.select_mask(Esum, tau, out=msk).float().mean().item()))
        for tau in taus:
            counts.zero_()
            e0, e1 = ev(), ev()
            e0.record(st)
            ops.select_mask_batched(E_all[t * n_in:(t + 1) * n_in], [tau] * n_in, count_accum=counts,
                                    write_masks=False)
            e1.record(st)
            vote = ops.aggregate_masks(counts, n_in, (1, 2))
            torch.cuda.synchronize()
            sel_ms.append(e0.elapsed_time(e1))
            dens["vote"][str(tau)].append(float(vote.float().mean().item()))
        del qk
    tau_of = lambda t: 0.99 if t < T // 3 else (0.95 if t < 2 * T // 3 else 0.9)
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev)
    sel_all = select_leg(E_all, [tau_of(t) for t in range(T) for _ in range(n_in)], torch, ops, flush, peaks)
    del E_all, flush
    # the dictionary of the sweep: one slice per timestep with a stricter tau early on
    # (tau(t) = 0.99, 0.95, 0.9 over the three thirds of the schedule), repetition
    # detection at gamma = 0.9 and stride 4, built by the calibration driver, saved, reloaded
    from calibrated_block_sparse_calib_b200.calibrate import calibrate_slice
    from calibrated_block_sparse_calib_b200.dictionary import MaskDictionary
    import tempfile
    dct = MaskDictionary(T, 1, H, nb, nb, B, stride=4, rho=(1, 2), mode="vote", n_inputs=n_in, gamma=0.9)
    members = torch.from_numpy(synth.sample_video_tokens(s, 512, seed=3)).to(dev)
    t_d = time.perf_counter()
    flags = []
    for t in range(T):
        tau_t = tau_of(t)
        qk = [synth.make_qkv(wl, input_idx=d, device=dev, pos_scale=1.0 + 0.125 * t)[:2] for d in range(n_in)]
        mask_t, rep_t, _ = calibrate_slice(qk, s.F, s.Hl, s.Wl, 0, B, tau_t, (1, 2), "vote", 0.9, 4, members)
        dct.put_mask(t, 0, mask_t, rep_t, tau=tau_t)
        flags.append(sum(rep_t))
        del qk
    torch.cuda.synchronize()
    build_s = time.perf_counter() - t_d
    with tempfile.TemporaryDirectory() as td:
        path = os.path.join(td, "sweep.cbsd")
        dct.save(path)
        file_bytes = os.path.getsize(path)
        back = MaskDictionary.load(path)
        same = all(torch.equal(back.block_list(t, 0).col_idx, dct.block_list(t, 0).col_idx) for t in range(T))
    ops.device_check()
    em = statistics.median(e_ms)
    sm_ = statistics.median(sel_ms)
    sel_bytes = n_in * H * nb * nb * 4 + H * nb * nb * 8   # 4 inputs' energies in, vote counts read + written
    exps = 2.0 * N * N * H / (em * 1e-3)
    peak = MUFU_EX2_PER_CLK_SM * B200_SMS * 1965.0e6
    print(json.dumps({
        "leg": "calibration_sweep", "workload": wl.name, "H": H, "N": N, "block": B, "inputs": n_in,
        "timesteps": T, "taus": list(taus), "energy_passes": len(e_ms) + len(a_ms),
        "energy_ms_median": em, "energy_exp2_per_s": exps, "energy_frac_of_mufu_at_1965mhz": exps / peak,
        "energy_tflops_qk": 2 * 2.0 * N * N * s.D * H / (em * 1e-3) / 1e12,
        "energy_accumulate_ms_median": statistics.median(a_ms),
        "select_vote_launch_ms_median": sm_, "select_vote_launch_gbs": sel_bytes / (sm_ * 1e-3) / 1e9,
        "select_all_entries": sel_all,
        "kept_density": dens,
        "dictionary": {"slices": T, "tau_schedule": [0.99 if t < T // 3 else (0.95 if t < 2 * T // 3 else 0.9)
                                                     for t in range(T)],
                       "repeat_heads_per_timestep": flags, "build_s": build_s, "file_bytes": file_bytes,
                       "reload_identical": bool(same)},
        "wall_s": time.perf_counter() - t_start}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="wan13b", choices=["wan13b", "wan14b720p", "mochi1"])
    ap.add_argument("--timestep", type=int, default=0, help="timestep of the mask schedule (mochi1)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip dense / e2e / calibration / other-config legs")
    ap.add_argument("--no-configs", action="store_true", help="skip the Wan-14B / Mochi-1 legs")
    ap.add_argument("--energy-only", action="store_true",
                    help="time only the fused LSE + block-energy pass (calibration) and print its own line")
    ap.add_argument("--heads", type=int, default=None, help="with --energy-only: the first H heads only")
    ap.add_argument("--calibration-sweep", action="store_true",
                    help="the calibration sweep: energies + selection over 4 inputs x 8 timesteps x 3 taus, "
                         "cross-input vote and energy-mean modes; prints its own line")
    ap.add_argument("--ref-seconds", type=float, default=60.0,
                    help="--impl reference: total seconds of oracle work over the timed steps")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist
    from calibrated_block_sparse_calib_b200 import ops, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    ops.lib()

    wl = synth.WORKLOADS[args.workload]
    s = wl.shape
    B, D, N, H = s.block, s.D, s.N, s.H
    if args.energy_only:
        return run_energy_only(args, wl, dev, torch, ops, synth)
    if args.calibration_sweep:
        return run_calibration_sweep(dev, torch, ops, synth)
    q, k, v = synth.make_qkv(wl, device=dev)
    mask_np = synth.make_head_masks(wl, timestep=args.timestep)
    mask = torch.from_numpy(mask_np).to(dev)
    bl = ops.BlockList.from_mask(mask, B)
    rep = [h in wl.repeat_heads for h in range(H)]
    stride = wl.repeat_stride
    n_anchor = ops.anchor_count(s.F, s.Hl, s.Wl, s.n_text, stride) if any(rep) else None
    out = torch.empty_like(q)
    if any(rep):
        call = lambda: ops.sparse_attn_fwd_repeat(q, k, v, bl, rep, s.F, s.Hl, s.Wl, s.n_text, stride, out=out)
    else:
        call = lambda: ops.sparse_attn_fwd(q, k, v, bl, out=out)
    flops_kept = kept_flops(mask_np, N, D, B, tuple(h for h in range(H) if rep[h]), n_anchor)
    flops_dense = 4.0 * N * N * D * H
    density = flops_kept / flops_dense
    ops.device_check()

    # ---- timed region: K inference calls ----------------------------------------
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
    gpu_id = gpu_uuid if gpu_uuid.startswith("GPU-") else f"GPU-{gpu_uuid}"
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_id) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record(st)
        for _ in range(args.steps):
            call()
        e1.record(st)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    ops.device_check()
    ms = e0.elapsed_time(e1) / args.steps
    if world > 1:
        ms = max_over_ranks(ms, dist, dev)
    value = whole_job_tflops(flops_kept, world, ms)
    peaks = _peaks()

    extras = {}
    if not args.no_extras:
        # own dense kernel: same pipeline, all-kept list
        full = torch.ones_like(mask)
        bl_dense = ops.BlockList.from_mask(full, B)
        ms_dense = _time_calls(lambda: ops.sparse_attn_fwd(q, k, v, bl_dense, out=out), 10, 3, torch)
        extras["dense_kernel"] = {"ms": ms_dense, "tflops": flops_dense / (ms_dense * 1e-3) / 1e12,
                                  "speedup_sparse_vs_dense": ms_dense / ms}
        # density sweep on the same shapes (seeded generator masks), against the dense kernel
        if wl.name == "wan13b" and not any(rep):
            sweep = {}
            for d in (0.10, 0.20, 0.30, 0.50):
                m_d = synth.make_head_masks(wl, density=d)
                bl_d = ops.BlockList.from_mask(torch.from_numpy(m_d).to(dev), B)
                fk = kept_flops(m_d, N, D, B)
                ms_d = _time_calls(lambda: ops.sparse_attn_fwd(q, k, v, bl_d, out=out), 20, 3, torch)
                sweep[f"{d:.2f}"] = {"density": round(fk / flops_dense, 4), "ms": ms_d,
                                     "kept_tflops": fk / (ms_d * 1e-3) / 1e12,
                                     "dense_equiv_tflops": flops_dense / (ms_d * 1e-3) / 1e12,
                                     "frac_of_bf16_peak": fk / (ms_d * 1e-3) / 1e12 / peaks["bf16_tflops"],
                                     "speedup_vs_dense": ms_dense / ms_d}
            sweep["1.00"] = {"density": 1.0, "ms": ms_dense, "kept_tflops": flops_dense / (ms_dense * 1e-3) / 1e12,
                             "dense_equiv_tflops": flops_dense / (ms_dense * 1e-3) / 1e12,
                             "frac_of_bf16_peak": flops_dense / (ms_dense * 1e-3) / 1e12 / peaks["bf16_tflops"],
                             "speedup_vs_dense": 1.0}
            extras["density_sweep"] = sweep
        # end to end through the public API with host buffers
        qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
        oh = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        qd, kd, vd = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

        def e2e_step():
            qd.copy_(qh, non_blocking=True)
            kd.copy_(kh, non_blocking=True)
            vd.copy_(vh, non_blocking=True)
            if any(rep):
                ops.sparse_attn_fwd_repeat(qd, kd, vd, bl, rep, s.F, s.Hl, s.Wl, s.n_text, stride, out=out)
            else:
                ops.sparse_attn_fwd(qd, kd, vd, bl, out=out)
            oh.copy_(out, non_blocking=True)

        ms_serial = _time_calls(e2e_step, 10, 3, torch)
        if world > 1:
            ms_serial = max_over_ranks(ms_serial, dist, dev)
        nb = q.numel() * q.element_size()
        # sparse_attn_fwd_host: per chunk of 3 heads (the last chunk's heads one at a time), the
        # host -> device copies of the next chunk and the device -> host copy of the previous
        # one overlap the attention
        hpc = 3
        staging = ops.HostStaging(qd, kd, vd, out)
        geom = (rep, s.F, s.Hl, s.Wl, s.n_text, stride) if any(rep) else None
        ms_e2e = _time_calls(lambda: ops.sparse_attn_fwd_host(qh, kh, vh, bl, staging=staging, out=oh,
                                                              heads_per_chunk=hpc, repeat=geom), 10, 3, torch)
        if world > 1:
            ms_e2e = max_over_ranks(ms_e2e, dist, dev)
        mode = "sparse_attn_fwd_host: copies overlapped with the attention per head chunk"
        extras["e2e"] = {"value": flops_kept * world / (ms_e2e * 1e-3) / 1e12, "unit": UNIT,
                         "h2d_bytes_per_step": 3 * nb, "d2h_bytes_per_step": nb, "ms_per_step": ms_e2e,
                         "mode": mode, "heads_per_chunk": hpc,
                         "serial_copies_value": flops_kept * world / (ms_serial * 1e-3) / 1e12}
        # calibration rows on the same shapes: fused LSE + energy pass and selection
        if wl.name == "wan13b":
            energy = ops.block_energy(q, k, B)
            ms_energy = _time_calls(lambda: ops.block_energy(q, k, B, out=energy), 3, 2, torch)
            msk = torch.empty(energy.shape, dtype=torch.uint8, device=dev)
            ms_sel = _time_graph(lambda: ops.select_mask(energy, 0.95, out=msk), 20, torch)
            sel_bytes = energy.numel() * 4 + msk.numel()
            # the calibration sweep's shape: 4 inputs x 8 timesteps of these energies in one
            # launch (each entry its own copy in HBM, tau(t) per timestep), L2 flushed before
            # every launch
            flush = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev)
            batch = energy.unsqueeze(0).repeat(32, 1, 1, 1)
            taus32 = [0.99 if t < 3 else (0.95 if t < 6 else 0.9) for t in range(8) for _ in range(4)]
            sel_batched = select_leg(batch, taus32, torch, ops, flush, peaks)
            del batch
            # LSE reuse: a dense forward that emits the row LSE (calibration runs the dense
            # model anyway), then the energy pass with that LSE runs a single pass
            lse_buf = torch.empty((H, N), dtype=torch.float32, device=dev)
            ms_attn_lse = _time_calls(lambda: ops.sparse_attn_fwd(q, k, v, bl_dense, out=out, lse=lse_buf),
                                      5, 2, torch)
            ms_e1 = _time_calls(lambda: ops.block_energy(q, k, B, lse=lse_buf, out=energy), 5, 2, torch)
            exps = 2.0 * N * N * H / (ms_energy * 1e-3)
            clk_mhz = (clk.summary().get("sm_max_mhz") or 1965.0)
            mufu_peak = MUFU_EX2_PER_CLK_SM * B200_SMS * clk_mhz * 1e6
            extras["calibration"] = {
                "energy_ms": ms_energy,
                "energy_tflops_qk": 2 * 2.0 * N * N * D * H / (ms_energy * 1e-3) / 1e12,
                "energy_exps_per_s": exps,
                "energy_with_attention_lse": {"dense_fwd_with_lse_ms": ms_attn_lse, "energy_one_pass_ms": ms_e1,
                                              "exp2_per_s": N * N * H / (ms_e1 * 1e-3)},
                "energy_roofline": {"bound": "alu", "unit": "exp2/s", "achieved": exps, "peak": mufu_peak,
                                    "frac": exps / mufu_peak, "kernel": f"block_energy_kernel<{D},{B},4>",
                                    "peak_source": "16 MUFU ex2 per clock per SM x 148 SMs x max SM clock"},
                "select_ms": ms_sel, "select_gbs": sel_bytes / (ms_sel * 1e-3) / 1e9,
                "select_frac_hbm": sel_bytes / (ms_sel * 1e-3) / 1e9 / peaks["hbm_gbs"],
                "tau": 0.95, "selected_density": float(msk.float().mean().item()),
                "select_batched_32": sel_batched}
            # spatial-repetition detection: cosine of 1024 sampled tokens' attention rows
            # against their stride-4 anchors, two passes over K, then the per-head decision
            mem = torch.from_numpy(synth.sample_video_tokens(s, 1024, seed=1)).to(dev)
            cos = ops.repeat_similarity(q, k, mem, s.F, s.Hl, s.Wl, 4)
            ms_sim = _time_calls(lambda: ops.repeat_similarity(q, k, mem, s.F, s.Hl, s.Wl, 4), 3, 1, torch)
            mean, flag = ops.repeat_flags(cos, mem, s.F, s.Hl, s.Wl, 4, 0.9)
            rows_sim = 2 * 2 * mem.numel()          # anchor + sample rows, two passes
            extras["calibration"]["repeat_detection"] = {
                "samples": mem.numel(), "stride": 4, "gamma": 0.9, "ms": ms_sim,
                "tflops_qk": 2.0 * rows_sim * N * D * H / (ms_sim * 1e-3) / 1e12,
                "mean_similarity_min": float(mean.min().item()), "mean_similarity_max": float(mean.max().item()),
                "heads_flagged": int(flag.sum().item())}
            # interval form of the default workload's skip list (mask storage)
            rows = H * s.nblk
            iv = ops.csr_to_intervals(bl.row_ptr, bl.col_idx, H, s.nblk)
            # the raw ABI call on the current stream (the binding's wrapper reads the run count
            # back to the host, which a graph capture does not allow)
            ms_enc = _time_graph(lambda: ops.lib().calib_csr_to_intervals(
                bl.row_ptr.data_ptr(), bl.col_idx.data_ptr(), H, s.nblk, iv[0].data_ptr(),
                iv[1].data_ptr(), iv[2].data_ptr(), torch.cuda.current_stream().cuda_stream), 20, torch)
            nnz, n_iv = int(bl.row_ptr[-1].item()), int(iv[0][-1].item())
            extras["calibration"]["skip_list_intervals"] = {
                "kept_blocks": nnz, "runs": n_iv, "blocks_per_run": nnz / max(1, n_iv),
                "csr_bytes": 4 * (rows + 1) + 2 * nnz, "interval_bytes": 4 * (rows + 1) + 4 * n_iv,
                "encode_ms": ms_enc}
            ops.device_check()

    # the other model-shaped workloads, each under its own clock record (replica 0 of a
    # multi-GPU run measures them; the others wait at the final barrier)
    if not args.no_extras and not args.no_configs and wl.name == "wan13b" and rank == 0:
        flush = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev)
        extras["configs"] = {
            "wan14b720p": config_leg("wan14b720p", synth.WORKLOADS["wan14b720p"], 0, dev, torch, ops, synth, peaks,
                                     steps=10, dense_iters=2, flush=flush, with_select=True),
            "mochi1_t0": config_leg("mochi1", synth.WORKLOADS["mochi1"], 0, dev, torch, ops, synth, peaks,
                                    steps=20, dense_iters=2),
            "mochi1_t7": config_leg("mochi1", synth.WORKLOADS["mochi1"], 7, dev, torch, ops, synth, peaks,
                                    steps=20, dense_iters=0),
        }
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(wl, mask_np, world, n_anchor),
        "dense_equiv_tflops": flops_dense * world / (ms * 1e-3) / 1e12,
        "frac_of_bf16_peak": value / world / peaks["bf16_tflops"],
        "roofline": {"bound": "tensor", "achieved": value / world, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": value / world / peaks["bf16_tflops"],
                     "traffic": NCU_TRAFFIC.get((wl.name, _src_sha("attn_fwd.cuh"), _src_sha("ptx.cuh"))),
                     "algorithmic_bytes": 4 * q.numel() * q.element_size(),
                     "peak_source": f"{peaks['source']} bf16 burst", "kernel": f"attn_fwd_kernel<{D},{B},3,2,0>",
                     "frac_of_sustained": value / world / peaks["bf16_tflops_sustained"]},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
    }
    if "e2e" in extras:
        line["e2e"] = extras.pop("e2e")
    line.update(extras)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, q, k, v, mask_np)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
