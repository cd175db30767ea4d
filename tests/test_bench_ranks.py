"""Multi-rank host logic of bench.py, on CPU with the gloo backend (world size 2).

The data path shards by request (each rank runs its own replica of the
workload, no collective), so the only cross-rank steps are the timing
reduction and the whole-job rate. These tests run them in two gloo ranks and
check the reference arm's rank-0-only rule.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took (r + 1) * 10 ms; the job took as long as the slowest rank
        ms = bench.max_over_ranks((rank + 1) * 10.0, dist, torch.device("cpu"))
        rate = bench.job_rate(1000, world, ms)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms": ms, "rate": rate}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_gloo(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["ms"] == 20.0  # both ranks see the max, not their own time
        assert r["rate"] == pytest.approx(1000 * world / 0.020)


def test_job_rate_is_weak_scaling():
    assert bench.job_rate(5, 1, 1.0) == pytest.approx(5000.0)
    assert bench.job_rate(5, 8, 1.0) == pytest.approx(8 * 5000.0)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_append_stats_closed_form():
    # 32 requests x 1 token of INT4/INT4 g64: 1152 B read + 324 B written per token
    from bit_mla_kv_qdecode_b200 import synth
    a = bench.append_stats(synth.workload("dsv3"), 0.01)
    assert a["tokens"] == 32 and a["bytes"] == 32 * (1152 + 324)
    assert abs(a["tokens_per_s"] - 3.2e6) < 1e-3 and abs(a["gbs"] - 32 * 1476 / 1e-5 / 1e9) < 1e-9
    m = bench.append_stats(synth.workload("mtp"), 0.02)  # INT2 g32 content: 228 B per token, 2 tokens each
    assert m["tokens"] == 256 and m["bytes"] == 256 * (1152 + 228)
