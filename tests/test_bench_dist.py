"""The multi-process side of bench.py on CPU (gloo, world size 2).

bench.py --gpus N runs one replica of the workload per GPU under torchrun:
every rank times its own steps, the time reported is the max over ranks, the
throughput is the whole job's, and only rank 0 prints.  These tests run that
host logic with two gloo ranks on this machine, and check that the reference
arm (the CPU oracle) runs on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slower one
        worst = bench.ranks_max(local_ms, world, dist, "cpu")
        value = bench.job_throughput(world, 32760, worst / 50)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"worst": worst, "value": value}, f)
    finally:
        dist.destroy_process_group()


def test_ranks_agree_on_the_slowest_time_and_the_whole_job_throughput(tmp_path):
    import torch.multiprocessing as mp
    mp.start_processes(_rank_main, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    assert res[0] == res[1]
    assert res[0]["worst"] == 15.0
    # 2 replicas x 32760 tokens in 15 ms / 50 steps per step
    assert res[0]["value"] == pytest.approx(2 * 32760 / (0.3e-3) / 1e6)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.ranks_max(3.5, 1) == 3.5
    assert bench.job_throughput(1, 1000, 1.0) == pytest.approx(1.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
