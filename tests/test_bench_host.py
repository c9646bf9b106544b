"""Host-side logic of bench.py that needs no GPU: the multi-rank reduction (two gloo ranks on
CPU, as torchrun would launch them), the whole-job aggregation of replicas, and the
reference arm (the float64 oracle on the host, rank 0 only)."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, dist, torch.device("cpu"))
        out[rank] = (ms, bench.whole_job_tflops(2.0e12, world, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_gloo():
    world = 2
    port = 29500 + os.getpid() % 1000
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    # every rank sees the slowest rank's time; the value counts both replicas' work
    assert res[0][0] == res[1][0] == 15.0
    assert res[0][1] == pytest.approx(2 * 2.0e12 / 15e-3 / 1e12)


def _run_bench(args, env_extra):
    env = dict(os.environ)
    env.update(env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True,
                          text=True, env=env, timeout=600)


def test_reference_arm_nonzero_rank_exits_without_work():
    r = _run_bench(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"],
                   {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_prints_one_json_line():
    r = _run_bench(["--impl", "reference", "--steps", "2", "--warmup", "3", "--ref-seconds", "2"],
                   {"RANK": "0", "WORLD_SIZE": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "TFLOPS"
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["workload"] == "wan13b"


def test_warmup_below_three_is_rejected():
    r = _run_bench(["--impl", "reference", "--steps", "1", "--warmup", "2"], {"RANK": "0"})
    assert r.returncode != 0
