"""The multi-process paths of ``bench.py`` on the CPU, with the gloo backend and two ranks.

The hot path has no exchange (every rank runs the whole workload on its own GPU), so what runs on
several ranks is plumbing: a barrier around the timed region, the maximum over ranks of the device
times, the whole-job rate computed from it, and the reference arm, which rank 0 alone runs under
torchrun while the other ranks exit 0. All rendezvous use 127.0.0.1.
"""
import datetime
import json
import os
import socket
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench

    ranks = bench.Ranks(world, torch.device("cpu"))
    ranks.barrier()
    # each rank's "device times": the max over ranks is taken element by element
    got = ranks.max([float(rank + 1), 10.0 - rank, -float(rank)])
    ranks.barrier()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(got, f)
    dist.destroy_process_group()


def test_max_over_ranks_with_gloo(tmp_path):
    import torch.multiprocessing as mp

    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        with open(tmp_path / f"rank{r}.json") as f:
            assert json.load(f) == [2.0, 10.0, 0.0], r


def test_single_rank_plumbing_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    ranks = bench.Ranks(1, torch.device("cpu"))
    ranks.barrier()
    assert ranks.max([3.0, -1.0]) == [3.0, -1.0]


def test_whole_job_rate_counts_every_rank_over_the_slowest():
    sys.path.insert(0, ROOT)
    import bench

    # two ranks, 100 units each, slowest rank 4 s -> 50 units/s for the job
    assert bench.whole_job_rate(2, 100.0, 4.0) == 50.0
    assert bench.whole_job_rate(1, 100.0, 4.0) == 25.0


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(ln) for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
