"""A plain C program compiled against include/streaming_top.h calls the
host-buffer entry point si_indexer_topk_host: it builds and links on the CPU,
refuses a bad argument there without touching CUDA, and on a B200 returns
the oracle's rows bit for bit on integer inputs."""
import os
import subprocess

import numpy as np
import pytest

import oracle
import synth
from tests import parity

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c", "host_api_main.c")
LIBDIR = os.path.join(ROOT, "streaming_top_b200")


@pytest.fixture(scope="module")
def c_program(tmp_path_factory):
    exe = str(tmp_path_factory.mktemp("capi") / "host_api_main")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-O2", "-I", os.path.join(ROOT, "include"),
                    SRC, "-L", LIBDIR, "-lstreaming_top", f"-Wl,-rpath,{LIBDIR}", "-o", exe], check=True)
    return exe


def _write_problem(path, hdr, q, kc, w):
    with open(path, "wb") as f:
        f.write(np.asarray(hdr, np.int32).tobytes())
        f.write(q.astype(np.uint16).tobytes())
        f.write(kc.astype(np.uint16).tobytes())
        f.write(w.astype(np.float32).tobytes())


def _read_result(path, n):
    raw = open(path, "rb").read()
    st = int(np.frombuffer(raw[:4], np.int32)[0])
    idx = np.frombuffer(raw[4:4 + 4 * n], np.int32)
    sc = np.frombuffer(raw[4 + 4 * n:4 + 8 * n], np.float32)
    return st, idx, sc


def test_c_caller_builds_and_a_bad_argument_is_refused_on_the_host(c_program, tmp_path):
    """k = 0 is refused by host-side validation (SI_ERR_INVALID_ARGUMENT = 1)
    before any CUDA call, so this runs without a GPU."""
    B, R, T, H, D = 1, 8, 2, 64, 128
    q = np.zeros((B, R, H, D), np.uint16)
    kc = np.zeros((B, T, D), np.uint16)
    w = np.zeros((B, R, H), np.float32)
    _write_problem(tmp_path / "in.bin", [B, R, T, H, D, 4, 0, 0, 0], q, kc, w)
    r = subprocess.run([c_program, str(tmp_path / "in.bin"), str(tmp_path / "out.bin")], capture_output=True)
    assert r.returncode == 1
    st, _, _ = _read_result(tmp_path / "out.bin", 0)
    assert st == 1, r.stderr


@pytest.mark.gpu
@pytest.mark.parametrize("B,S,T,k,row0,chunk", [
    (1, 2048, 512, 128, 0, 0),        # one chunk (default size)
    (2, 1030, 256, 96, 0, 256),       # five chunks, the last ragged; two sequences
    (1, 1500, 512, 64, 548, 512),     # rows 548 .. 2047 of a longer sequence
])
def test_c_caller_matches_the_oracle(c_program, tmp_path, B, S, T, k, row0, chunk):
    R = S - row0
    H, D, m = 64, 128, 4
    seed = 61 + S + row0
    q = synth.matrix(B * S * H, D, seed, synth.TENSOR_Q, "int").reshape(B, S, H, D)
    kc = synth.matrix(B * T, D, seed, synth.TENSOR_KC, "int").reshape(B, T, D)
    w = synth.weights(B * S * H, seed, synth.TENSOR_W, "pow2").reshape(B, S, H)
    _write_problem(tmp_path / "in.bin", [B, R, T, H, D, m, k, row0, chunk], q[:, row0:], kc, w[:, row0:])
    r = subprocess.run([c_program, str(tmp_path / "in.bin"), str(tmp_path / "out.bin")], capture_output=True)
    assert r.returncode == 0, r.stderr.decode()
    st, idx, sc = _read_result(tmp_path / "out.bin", B * R * k)
    assert st == 0
    rows = np.concatenate([np.arange(row0, S) + b * S for b in range(B)])
    oi, osc, _ = oracle.topk(q, kc, w, m, k, rows=rows)
    parity.compare_exact(idx.reshape(-1, k), sc.reshape(-1, k), oi, osc, rows)
