"""Split-key streaming (the causal chunk driver's split of long rows over
keys): a row-range call with too few query rows to give every SM a unit
splits each unit's keys over CTAs, each CTA keeps its partition's exact
top-k, and a merge kernel selects the rows' top-k (StreamIndex's
partition-merge).  Checked bit for bit against the oracle and against the
same rows computed without a split, on integer inputs; on planted Gaussian
inputs within the tolerance and on plain recall."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity

pytestmark = pytest.mark.gpu

import streaming_top_b200 as si  # noqa: E402

T_LONG = 16384   # keys of the sequence (S = 4 T rows)
H, D, M = 64, 128, 4


def _int_rows(B, T, rows, seed):
    """Integer inputs (every score exact in fp32) of B sequences of 4T rows:
    q [B, 4T, H, D] lazily allocated with only `rows` generated (the others
    are never touched), kc and w complete."""
    S = M * T
    q = np.empty((B, S, H, D), np.uint16)
    for b in range(B):
        q[b, rows[0]:rows[-1] + 1] = synth.matrix_range((b * S + rows[0]) * H, len(rows) * H, D, seed,
                                                        synth.TENSOR_Q, "int", 1.0, "bf16").reshape(-1, H, D)
    kc = synth.matrix(B * T, D, seed, synth.TENSOR_KC, "int").reshape(B, T, D)
    w = synth.weights(B * S * H, seed, synth.TENSOR_W, "pow2").reshape(B, S, H)
    return q, kc, w


def _dev(q, kc, w):
    return (torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).cuda(),
            torch.from_numpy(kc.view(np.int16)).view(torch.bfloat16).cuda(), torch.from_numpy(w).cuda())


@pytest.mark.parametrize("B,R,k,kw", [
    (1, 4, 512, {}),                       # one unit over ~all SMs
    (1, 16, 512, {}),
    (1, 64, 512, {}),                      # 16 units, 9 partitions each
    (2, 6, 300, {}),                       # two sequences, a ragged unit
    (1, 8, 2048, {"key_tile": 128}),       # k = 2048
    (1, 8, 100, {"key_tile": 64}),         # 64-key partitions of the partition-merge
])
def test_split_rows_equal_unsplit_rows_and_the_oracle(B, R, k, kw):
    S = M * T_LONG
    big0 = S - 640                         # 640 rows = 160 units per sequence: no split
    row0 = S - R - 37                      # the small call's rows lie inside the big call's
    q, kc, w = _int_rows(B, T_LONG, np.arange(big0, S), seed=90 + R + k)
    qd, kd, wd = _dev(np.ascontiguousarray(q[:, big0:]), kc, np.ascontiguousarray(w[:, big0:]))
    bi, bs = si.indexer_topk_rows(qd, kd, wd, M, k, big0, **kw)
    off = row0 - big0
    gi, gs = si.indexer_topk_rows(qd[:, off:off + R].contiguous(), kd, wd[:, off:off + R].contiguous(), M, k,
                                  row0, **kw)
    assert si.device_status() == si.SI_OK
    assert torch.equal(gi, bi[:, off:off + R]) and torch.equal(gs, bs[:, off:off + R])
    rows = np.concatenate([b * S + np.arange(row0, row0 + R) for b in range(B)])
    oi, osc, _ = oracle.topk(q, kc, w, M, k, rows=rows)
    parity.compare_exact(gi.cpu().numpy().reshape(-1, k), gs.cpu().numpy().reshape(-1, k), oi, osc, rows)


def test_split_rows_planted_gaussian():
    """The v4flash recipe's planted inputs at the sequence's end: 16 rows split
    over the SMs, checked against the oracle on score tolerance, the tie
    window and plain recall."""
    wl = synth.WORKLOADS["v4flash"]
    R = 16
    row0 = wl.S - R
    rows = np.arange(row0, wl.S)
    inp = synth.make_inputs_rows(wl, rows)
    q = np.ascontiguousarray(inp["q"][:, row0:])
    w = np.ascontiguousarray(inp["w"][:, row0:])
    qd, kd, wd = _dev(q, inp["kc"], w)
    gi, gs = si.indexer_topk_rows(qd, kd, wd, wl.m, wl.k, row0)
    assert si.device_status() == si.SI_OK
    gi, gs = gi.cpu().numpy().reshape(-1, wl.k), gs.cpu().numpy().reshape(-1, wl.k)
    oi, _, osc64 = oracle.topk(inp["q"], inp["kc"], inp["w"], wl.m, wl.k, rows=rows)
    parity.check_structure(gi, gs, rows, wl.S, wl.T, wl.m)
    st = parity.compare_tolerant(gi, gs, oi, osc64, rows,
                                 lambda r: oracle.scores(inp["q"], inp["kc"], inp["w"], wl.m, r))
    parity.report("workload_recall", "v4flash_split_rows", {"stream_vs_oracle": st})
    parity.assert_recall((st, "split rows vs oracle"))


def test_split_rows_fp8():
    """e4m3 inputs through the split path equal the unsplit rows."""
    wl = synth.WORKLOADS["v4flash"]
    S, T = wl.S, wl.T
    big0, R = S - 640, 12
    inp = synth.make_inputs(wl, fmt="e4m3", S=S, skip_q=True)
    q8, qsc = synth.q_rows(wl, 0, big0, S - big0, "e4m3")
    qd = torch.from_numpy(np.ascontiguousarray(q8[None])).cuda()
    qsd = torch.from_numpy(np.ascontiguousarray(qsc[None])).cuda()
    kd, ksd = torch.from_numpy(inp["kc"]).cuda(), torch.from_numpy(inp["kc_scale"]).cuda()
    wd = torch.from_numpy(np.ascontiguousarray(inp["w"][:, big0:])).cuda()
    bi, bs = si.indexer_topk_rows(qd, kd, wd, wl.m, wl.k, big0, q_scale=qsd, kc_scale=ksd)
    off = 640 - R
    si_, ss = si.indexer_topk_rows(qd[:, off:].contiguous(), kd, wd[:, off:].contiguous(), wl.m, wl.k, big0 + off,
                                   q_scale=qsd[:, off:].contiguous(), kc_scale=ksd)
    assert si.device_status() == si.SI_OK
    assert torch.equal(si_, bi[:, off:]) and torch.equal(ss, bs[:, off:])
    assert T == kd.shape[1]
