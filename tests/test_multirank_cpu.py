"""Host logic of the multi-rank bench path, run as two gloo ranks on CPU.

Every rank runs independent sequences of its own (no data exchange); the only
collective is the max-over-ranks of the measured times.  These tests check
that logic without a GPU: per-rank seeds give different inputs of the same
shape, the max reduction returns the slowest rank's time on every rank, and
the whole-job value counts every rank's pairs over that time.  The reference
arm does its work on rank 0 only.
"""
from __future__ import annotations

import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = synth.WORKLOADS["tiny"]
        seed = bench.rank_seed(wl, rank)
        inp = synth.make_inputs(wl, seed=seed, S=64)
        slowest = bench.max_over_ranks(times[rank], torch.device("cpu"))
        np.save(os.path.join(out_dir, f"q{rank}.npy"), inp["q"])
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(f"{seed} {slowest!r}\n")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_seed_and_max(tmp_path):
    world, times = 2, [3.25, 7.5]
    mp.start_processes(_rank_main, args=(world, _free_port(), times, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    seeds, slow = [], []
    for r in range(world):
        a, b = open(tmp_path / f"r{r}.txt").read().split()
        seeds.append(int(a))
        slow.append(float(b))
    assert slow == [max(times)] * world
    assert len(set(seeds)) == world
    q0, q1 = np.load(tmp_path / "q0.npy"), np.load(tmp_path / "q1.npy")
    assert q0.shape == q1.shape and not np.array_equal(q0, q1)


def test_job_value_counts_all_ranks():
    P = synth.WORKLOADS["v4flash"].visible_pairs()
    assert bench.job_value(1, P, 10.0) == pytest.approx(P / 0.01)
    assert bench.job_value(4, P, 10.0) == pytest.approx(4 * bench.job_value(1, P, 10.0))


def test_reference_arm_nonzero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "tiny"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
