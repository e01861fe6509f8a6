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


def _rows_rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import streaming_top_b200 as si
        wl = synth.WORKLOADS["tiny"]
        S, m, k = 512, wl.m, 24
        T = S // m
        bounds = si.row_shards(S, T, m, world)
        r0, r1 = bounds[rank], bounds[rank + 1]
        # what a rank holds in the row-sharded bench: its own q rows, all keys
        # and the weights of the same sequence (the same seed on every rank)
        full = synth.make_inputs(wl, S=S)
        q_r = synth.q_rows(wl, 0, r0, r1 - r0, S=S)
        same_q = bool(np.array_equal(q_r, full["q"][0, r0:r1]))
        oi, osc, _ = oracle.topk(full["q"], full["kc"], full["w"], m, k, rows=np.arange(r0, r1))
        pairs = synth.visible_pairs(r1, T, m) - synth.visible_pairs(r0, T, m)
        got = [None] * world
        dist.all_gather_object(got, (bounds, same_q, pairs, oi, osc))
        if rank == 0:
            import pickle
            with open(os.path.join(out_dir, "rows.pkl"), "wb") as f:
                pickle.dump(got, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_row_shards(tmp_path):
    """Row sharding of one sequence: both ranks derive the same boundaries,
    the shards tile [0, S) with equal visible pairs, each rank's q rows
    generated alone equal that slice of the whole sequence's q, and the
    ranks' top-k rows put together are the whole sequence's."""
    import pickle

    import oracle
    world = 2
    mp.start_processes(_rows_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    got = pickle.load(open(tmp_path / "rows.pkl", "rb"))
    bounds = got[0][0]
    assert all(g[0] == bounds for g in got)
    assert bounds[0] == 0 and bounds[-1] == 512 and all(a < b for a, b in zip(bounds, bounds[1:]))
    assert all(g[1] for g in got)
    pairs = [g[2] for g in got]
    assert sum(pairs) == synth.visible_pairs(512, 128, 4)
    assert max(pairs) / min(pairs) < 1.03
    wl = synth.WORKLOADS["tiny"]
    full = synth.make_inputs(wl, S=512)
    ai, asc, _ = oracle.topk(full["q"], full["kc"], full["w"], 4, 24)
    assert np.array_equal(np.concatenate([g[3] for g in got]), ai)
    assert np.array_equal(np.concatenate([g[4] for g in got]), asc)


def test_row_shards_balance_and_cover():
    import streaming_top_b200 as si
    for S, T, m in [(65536, 16384, 4), (1048576, 262144, 4), (1000, 100, 4), (513, 171, 3)]:
        assert si.visible_pairs_before(S, T, m) == synth.visible_pairs(S, T, m)
        for parts in (1, 2, 4, 8):
            b = si.row_shards(S, T, m, parts)
            assert b[0] == 0 and b[-1] == S and len(b) == parts + 1
            assert all(x <= y for x, y in zip(b, b[1:]))
            assert all(x % 4 == 0 for x in b[1:-1])
            p = [si.visible_pairs_before(y, T, m) - si.visible_pairs_before(x, T, m) for x, y in zip(b, b[1:])]
            if S >= 65536:
                assert max(p) / min(p) < 1.001


def test_two_stage_pair_counts_match_brute_force():
    """bench's count of the pairs the two stages score (complete visible
    blocks, then kept blocks' keys plus the incomplete block's visible keys)
    against a row-by-row count, on a shape where the block budget binds."""
    import dataclasses
    wl = dataclasses.replace(synth.WORKLOADS["tiny"], S=70000)
    cp, fp = bench.two_stage_pairs(wl)
    G, keep = bench.TWO_STAGE["block"], bench.TWO_STAGE["n_keep"]
    c_bf = f_bf = 0
    for t in range(wl.S):
        n = min(wl.T, (t + 1) // wl.m)
        c_bf += n // G
        f_bf += min(n // G, keep) * G + n % G
    assert (cp, fp) == (c_bf, f_bf)
    assert fp < synth.visible_pairs(wl.S, wl.T, wl.m)


def test_reference_arm_two_stage_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--workload", "tiny", "--method", "two-stage", "--ref-rows", "8"],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    import json
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_bench_refuses_two_stage_with_other_formats():
    """The two-stage bench path runs bf16 inputs over whole sequences; other
    combinations are refused before any device work."""
    for extra in (["--fmt", "e4m3"], ["--shard", "rows"]):
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--method", "two-stage", "--workload",
                            "tiny", "--steps", "1", "--warmup", "0", *extra],
                           capture_output=True, text=True, timeout=300)
        assert r.returncode != 0 and "two-stage" in (r.stderr + r.stdout), (extra, r.stderr[-300:])
