"""The two-stage indexer (blocks of keys scored by their pooled key, the
best n_keep blocks kept, then the top-k of their keys) through the C ABI on
a B200, against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity

pytestmark = pytest.mark.gpu

import streaming_top_b200 as si  # noqa: E402  (fails loudly when the library is missing)


def _dev(inp):
    q = torch.from_numpy(inp["q"].view(np.int16)).view(torch.bfloat16).cuda()
    kc = torch.from_numpy(inp["kc"].view(np.int16)).view(torch.bfloat16).cuda()
    return q, kc, torch.from_numpy(inp["w"]).cuda()


def _int_inputs(B, S, T, seed, H=64, D=128):
    q = synth.matrix(B * S * H, D, seed, synth.TENSOR_Q, "int").reshape(B, S, H, D)
    kc = synth.matrix(B * T, D, seed, synth.TENSOR_KC, "int").reshape(B, T, D)
    w = synth.weights(B * S * H, seed, synth.TENSOR_W, "pow2").reshape(B, S, H)
    return {"q": q, "kc": kc, "w": w}


def _run(inp, m, k, **kw):
    q, kc, w = _dev(inp)
    idx, sc = si.indexer_topk_two_stage(q, kc, w, m, k, **kw)
    assert si.device_status() == si.SI_OK
    B, S = q.shape[:2]
    return idx.cpu().numpy().reshape(B * S, k), sc.cpu().numpy().reshape(B * S, k)


def test_all_blocks_kept_equals_one_stage():
    """Integer inputs with at most n_keep blocks: bit-exact against the
    streaming path and both oracles."""
    B, S, T, m, k = 1, 2048, 512, 4, 96
    inp = _int_inputs(B, S, T, seed=51)
    gi, gs = _run(inp, m, k, block=8, n_keep=64)
    q, kc, w = _dev(inp)
    ri, rs = si.indexer_topk(q, kc, w, m, k)
    assert np.array_equal(gi, ri.cpu().numpy().reshape(-1, k))
    assert np.array_equal(gs, rs.cpu().numpy().reshape(-1, k))
    oi, osc, _ = oracle.topk_two_stage(inp["q"], inp["kc"], inp["w"], m, k, G=8, n_keep=64)
    parity.compare_exact(gi, gs, oi, osc, np.arange(B * S))


@pytest.mark.parametrize("B,S,T,m,k,G,n_keep,chunk", [
    (1, 4096, 1024, 4, 64, 8, 16, 0),      # 128 blocks, 16 kept
    (2, 1030, 300, 3, 32, 4, 10, 300),     # m = 3, blocks of 4, odd rows, chunks of 300
    (1, 2048, 512, 4, 200, 8, 12, 1000),   # k > 8 * n_keep for late rows: candidates < k
    (1, 2048, 600, 4, 64, 6, 20, 0),       # blocks of 6: the cp.async gather (no whole TMA boxes)
    (1, 1024, 520, 2, 96, 16, 9, 0),       # blocks of 16: two 8-row boxes per block
])
def test_integer_two_stage_bit_exact(B, S, T, m, k, G, n_keep, chunk):
    """Integer inputs: pooled keys, coarse and fine scores are exact in fp32,
    so the block choice and the result match the oracle bit for bit."""
    inp = _int_inputs(B, S, T, seed=S + k + G)
    gi, gs = _run(inp, m, k, block=G, n_keep=n_keep, query_chunk=chunk)
    oi, osc, _ = oracle.topk_two_stage(inp["q"], inp["kc"], inp["w"], m, k, G=G, n_keep=n_keep)
    rows = np.arange(B * S)
    _check_two_stage_structure(gi, gs, S, T, m, G, n_keep)
    parity.compare_exact(gi, gs, oi, osc, rows)


def _check_two_stage_structure(gi, gs, S, T, m, G, n_keep):
    """Valid entries = min(k, candidates): the kept blocks' keys and the
    incomplete block's visible keys; then -1 / -inf; distinct, visible,
    sorted."""
    k = gi.shape[1]
    for r in range(gi.shape[0]):
        t = r % S
        n = min(T, (t + 1) // m)
        cand = min(n // G, n_keep) * G + n % G
        nv = min(k, cand)
        assert np.all(gi[r, :nv] >= 0) and np.all(gi[r, nv:] == -1), (r, nv)
        assert np.all(np.isneginf(gs[r, nv:])) and len(np.unique(gi[r, :nv])) == nv, r
        assert np.all(gi[r, :nv] < n), r
        assert np.all(np.diff(gs[r, :nv].astype(np.float64)) <= 0), r


def test_gaussian_two_stage_rows():
    """Planted Gaussian inputs (v4flash recipe, S = 65536, 2048 blocks of 8)
    with 256 kept blocks: on sampled rows every returned key comes from a
    block the oracle keeps or from one whose pooled score ties the n_keep-th
    within 1e-3, its score matches the oracle's, and every oracle key the GPU
    lacks is explained by such a block or by a fine tie."""
    wl = synth.WORKLOADS["v4flash"]
    G, n_keep, k, m = 8, 256, wl.k, wl.m
    inp = synth.make_inputs(wl)
    gi, gs = _run(inp, m, k, block=G, n_keep=n_keep)
    S, T = wl.S, wl.T
    rows = np.unique(np.concatenate([synth.sample_rows(30, m * G * (n_keep + 1), S, seed=7), [S - 1]]))
    pooled = synth.f32_to_bf16_bits(oracle.pool_keys(inp["kc"], G).astype(np.float32))
    oi, _, osc64 = oracle.topk_two_stage(inp["q"], inp["kc"], inp["w"], m, k, G=G, n_keep=n_keep, rows=rows)
    for n_r, r in enumerate(rows):
        coarse = oracle.scores(inp["q"], pooled, inp["w"], m * G, int(r))
        vis = np.nonzero(~np.isnan(coarse))[0]
        order = vis[np.lexsort((vis, -coarse[vis]))]
        kth = coarse[order[n_keep - 1]]
        tie = set(vis[np.abs(coarse[vis] - kth) <= 1e-3 * abs(kth)].tolist())
        kept = set(order[:n_keep].tolist())
        n = min(T, (int(r) + 1) // m)
        nbv = n // G
        fine = oracle.scores(inp["q"], inp["kc"], inp["w"], m, int(r))
        for j, x in enumerate(gi[r]):
            blk = x // G
            assert x < n and (blk >= nbv or blk in kept or blk in tie), (r, x)
            assert abs(gs[r, j] - fine[x]) <= 1e-3 * abs(fine[x]) + 1e-6, (r, x, gs[r, j], fine[x])
        kth_fine = osc64[n_r, k - 1]
        for x in set(oi[n_r].tolist()) - set(gi[r].tolist()):
            assert x // G in tie or abs(fine[x] - kth_fine) <= 1e-3 * abs(kth_fine), (r, x)
        assert np.all(np.diff(gs[r]) <= 0)
