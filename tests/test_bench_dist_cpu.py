"""bench.py's multi-rank logic on the CPU: two gloo ranks on 127.0.0.1.

Each rank times its own independent problem; the job's time is the slowest
rank's (max over ranks), the whole-job rate counts every rank's units, and
only rank 0 prints. The data path has no collective; these are the only ones.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [3.0, 5.0][rank]           # rank 1 is the slow one
        bench.barrier(world)
        ms = bench.max_over_ranks(local_ms, world)
        rate = bench.job_throughput(1000.0, ms, world)
        bench.barrier(world)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms": ms, "rate": rate}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_count_all_units(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    for r in range(world):
        d = json.load(open(tmp_path / f"rank{r}.json"))
        assert d["ms"] == pytest.approx(5.0)                 # max over ranks, on every rank
        assert d["rate"] == pytest.approx(1000.0 * 2 / 5e-3)  # both ranks' units / slowest time


def test_reference_arm_prints_only_on_rank_zero():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--ref-tokens", "64"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
