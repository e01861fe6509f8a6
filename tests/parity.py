"""Parity helpers: run the CPU oracle on rows (in a spawn process pool) and
compare the CUDA path's top-k against it.

Acceptance rules (the indexer top-k's contract):
  * integer-valued inputs: every score is exact in fp32, so indices and
    scores must match the oracle bit for bit;
  * Gaussian inputs:
      - the j-th returned score is within 1e-3 relative of the oracle's j-th
        score (absolute floor 1e-6 * the row's largest score);
      - every index that is in one set but not the other has an oracle score
        within a 1e-3 relative tie window of the oracle's k-th score;
      - set-overlap recall |G & O| / |O| -- plain, nothing counted as a hit
        that is not in both sets -- has mean >= 0.9999 and min >= 0.998 over
        the compared rows.
    A recall below that bar is a failure, with one exception that is
    reported as an expected failure (xfail), never as a pass: every key
    exchanged across the k-th place has an oracle score within
    FP32_EVAL_BOUND relative of the k-th score.  That bound is the textbook
    worst case of the fp32 evaluation of one score (a D-term dot product then
    an H_I-term weighted sum: (D + H_I) * 2^-24 relative), so the fp32 path
    cannot order such keys the way the fp64 oracle does.
  * always: valid entries = min(k, visible keys), -1 / -inf padding after
    them, distinct indices, every index causally visible, scores sorted
    descending.
"""
from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np

import oracle
import synth

REL = 1e-3
ABS_FLOOR = 1e-6
FP32_EVAL_BOUND = (128 + 64) * 2.0 ** -24
RECALL_MEAN = 0.9999
RECALL_MIN = 0.998


def _worker(args):
    wl_name, overrides, fmt, k, rows, sparse = args
    wl = synth.WORKLOADS[wl_name]
    if sparse:  # only this worker's q rows (a million-token q is 16 GiB)
        inp = synth.make_inputs_rows(wl, rows, fmt=fmt, **overrides)
    else:
        inp = synth.make_inputs(wl, fmt=fmt, **overrides)
    idx, sc, sc64 = oracle.topk(inp["q"], inp["kc"], inp["w"], wl.m, k, rows=rows,
                                q_scale=inp.get("q_scale"), kc_scale=inp.get("kc_scale"),
                                kc_mx_scale=inp.get("kc_mx_scale"))
    return idx, sc, sc64


def oracle_rows(wl_name: str, rows: np.ndarray, k: int, fmt: str = "bf16", overrides=None,
                procs: int | None = None, inputs=None, sparse: bool = False):
    """Oracle (idx, score, score64) for flat rows of a named workload.

    With `inputs` (the exact host arrays given to the GPU) it runs in this
    process; otherwise the rows are split over a spawn pool whose workers
    regenerate the same seeded inputs (with `sparse`, only the q rows they
    need)."""
    rows = np.asarray(rows, dtype=np.int64)
    wl = synth.WORKLOADS[wl_name]
    if inputs is not None:
        return oracle.topk(inputs["q"], inputs["kc"], inputs["w"], wl.m, k, rows=rows,
                           q_scale=inputs.get("q_scale"), kc_scale=inputs.get("kc_scale"),
                           kc_mx_scale=inputs.get("kc_mx_scale"))
    procs = procs or max(1, min(32, (os.cpu_count() or 2)))
    # interleave rows so every worker gets a similar mix of short and long rows
    parts = [rows[i::procs] for i in range(procs) if len(rows[i::procs])]
    ctx = mp.get_context("spawn")
    with ctx.Pool(len(parts)) as pool:
        res = pool.map(_worker, [(wl_name, overrides or {}, fmt, k, p, sparse) for p in parts])
    n = len(rows)
    idx = np.empty((n, k), np.int32)
    sc = np.empty((n, k), np.float32)
    sc64 = np.empty((n, k), np.float64)
    for i, (a, b, c) in enumerate(res):
        idx[i::len(parts)] = a
        sc[i::len(parts)] = b
        sc64[i::len(parts)] = c
    return idx, sc, sc64


def report(name: str, key: str, value) -> None:
    """Append a result to $SI_REPORT_DIR/<name>.json when that variable is set."""
    d = os.environ.get("SI_REPORT_DIR")
    if not d:
        return
    import json
    os.makedirs(d, exist_ok=True)
    path = os.path.join(d, f"{name}.json")
    data = json.load(open(path)) if os.path.exists(path) else {}
    data[key] = value
    json.dump(data, open(path, "w"), indent=1, sort_keys=True)


def check_structure(idx: np.ndarray, score: np.ndarray, rows: np.ndarray, S: int, T: int, m: int):
    """Padding, distinctness, causal visibility and order of GPU rows."""
    k = idx.shape[1]
    for r in range(len(rows)):
        t = int(rows[r]) % S
        n = min(T, (t + 1) // m)
        nv = min(k, n)
        ir = idx[r]
        assert np.all(ir[:nv] >= 0) and np.all(ir[nv:] == -1), (rows[r], ir[:8], nv)
        assert np.all(np.isneginf(score[r, nv:])), rows[r]
        assert len(np.unique(ir[:nv])) == nv, rows[r]
        assert np.all(ir[:nv] * m + m - 1 <= t), rows[r]
        assert np.all(np.diff(score[r, :nv].astype(np.float64)) <= 0.0), rows[r]


def compare_exact(gi, gs, oi, osc, rows):
    bad = np.nonzero(np.any(gi != oi, axis=1) | np.any(gs != osc, axis=1))[0]
    assert len(bad) == 0, (f"{len(bad)} rows differ; first row {rows[bad[0]]}: gpu {gi[bad[0], :8]} "
                           f"oracle {oi[bad[0], :8]}")


def compare_tolerant(gi, gs, oi, osc64, rows, score_row_fn) -> dict:
    """Asserts the score tolerance and the tie window row by row, and returns
    plain set-overlap recall: {"mean", "min", "rows", "swaps", "max_gap_rel"}.
    score_row_fn(row) -> oracle scores of all keys of that row (double), used
    only for rows with a mismatch; "swaps" counts the keys in one set but not
    the other, "max_gap_rel" their largest |score - k-th| / |k-th|."""
    recalls = []
    max_gap = 0.0
    swaps = 0
    for r in range(len(rows)):
        nv = int((oi[r] >= 0).sum())
        if nv == 0:
            assert np.all(gi[r] == -1)
            continue
        o = osc64[r, :nv]
        g = gs[r, :nv].astype(np.float64)
        floor = ABS_FLOOR * max(abs(o[0]), 1e-30)
        err = np.abs(g - o)
        assert np.all(err <= REL * np.abs(o) + floor), (rows[r], float(err.max()))
        G, O = set(gi[r, :nv].tolist()), set(oi[r, :nv].tolist())
        recalls.append(len(G & O) / nv)
        if G != O:
            allsc = score_row_fn(int(rows[r]))
            kth = o[-1]
            win = REL * abs(kth) + floor
            for x in G ^ O:
                gap = abs(allsc[x] - kth)
                assert gap <= win, (rows[r], x, allsc[x], kth)
                max_gap = max(max_gap, gap / max(abs(kth), 1e-30))
            swaps += len(G - O)
    rec = np.asarray(recalls) if recalls else np.ones(1)
    return {"mean": float(rec.mean()), "min": float(rec.min()), "rows": len(recalls),
            "swaps": swaps, "max_gap_rel": max_gap}


def assert_recall(*checks) -> None:
    """checks: (stats, label) pairs from compare_tolerant.  Plain recall must
    reach mean >= 0.9999 and min >= 0.998 in each.  A shortfall where every
    exchanged key lies within the fp32 evaluation bound of the k-th score is
    an expected failure (pytest.xfail with the figures, after all checks have
    been evaluated); any other shortfall fails."""
    soft, hard = [], []
    for stats, what in checks:
        if stats["mean"] >= RECALL_MEAN and stats["min"] >= RECALL_MIN:
            continue
        msg = (f"{what}: recall mean {stats['mean']:.6f} min {stats['min']:.6f} over {stats['rows']} rows; "
               f"{stats['swaps']} keys exchanged at the k-th place, largest gap "
               f"{stats['max_gap_rel']:.3g} relative to the k-th score")
        (soft if stats["max_gap_rel"] <= FP32_EVAL_BOUND else hard).append(msg)
    if hard:
        raise AssertionError("; ".join(hard + soft))
    if soft:
        import pytest
        pytest.xfail("; ".join(soft) + f" (all within the fp32 evaluation bound {FP32_EVAL_BOUND:.3g})")
