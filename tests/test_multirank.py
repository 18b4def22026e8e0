"""The N > 1 plumbing of bench.py on CPU ranks (gloo, world size 2): every rank runs its own
replica of the virtual ring (no data-path collective), the timing is the max over ranks, and the
job throughput sums the ranks' work over that time.  The reference arm runs on rank 0 only."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ms = [10.0, 17.5][rank]
    slowest = bench.max_over_ranks(ms, world, device="cpu")
    value = bench.job_throughput(1e12, world, slowest)
    dist.barrier()
    out[rank] = (slowest, value)
    dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, 29511, out), nprocs=world, join=True)
    for rank in range(world):
        slowest, value = out[rank]
        assert slowest == 17.5
        assert value == pytest.approx(2 * 1e12 / 17.5e-3 / 1e12)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0", "--ref-rows", "1"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "s4k", "--steps", "1", "--warmup", "0", "--ref-rows", "2"],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
