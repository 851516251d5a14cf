"""The benchmark's multi-GPU path on the CPU: two `gloo` ranks.

bench.py runs one full replica of the step per rank (the method needs no
exchange), takes the job time as the maximum of the ranks' device times and
reports the work of all replicas over it.  Here two processes stand in for
two GPUs: the max-over-ranks reduction and the throughput formula are checked
with times that differ per rank, and the reference arm runs on rank 0 only.
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


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_path):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = 10.0 + 5.0 * rank  # rank 1 is the slower replica
        job = bench.job_time_ms(local, world, dist, torch, torch.device("cpu"))
        tops = bench.job_tops(2.0e12, 4, job, world)
        with open(f"{out_path}.{rank}", "w") as f:
            json.dump({"job": job, "tops": tops}, f)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_throughput(tmp_path):
    world, port, out = 2, _free_port(), str(tmp_path / "r")
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    res = [json.load(open(f"{out}.{r}")) for r in range(world)]
    for r in res:
        assert r["job"] == 15.0  # the max of 10 and 15 ms, on every rank
        # 2 replicas x 2e12 ops x 4 steps over 15 ms
        assert r["tops"] == pytest.approx(2 * 2.0e12 * 4 / 15e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_time_ms(3.5, 1, None, torch, None) == 3.5
    assert bench.job_tops(1.0e12, 2, 4.0, 1) == pytest.approx(2 * 1.0e12 / 4e-3 / 1e12)


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "small",
           "--steps", "1", "--warmup", "0"]
    r1 = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=300)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    env0 = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r0 = subprocess.run(cmd, env=env0, capture_output=True, text=True, timeout=300)
    assert r0.returncode == 0
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_gpus_flag_starts_its_own_ranks():
    # `bench.py --gpus 2` without torchrun: the bench starts both ranks itself
    # (spawned processes with the environment torchrun would set); the
    # reference arm prints one line, from rank 0, with n_gpus = 2.
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "small",
           "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.strip().splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["config"]["parallelism"] == "replicas x2"
