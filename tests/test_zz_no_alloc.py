"""The allocation-free materialize entry point (collected last on purpose).

si_indexer_materialize_noalloc serves callers that cannot allocate device
memory during the call -- an application whose own pool already holds nearly
all GPU memory, a plugin step that must not allocate, a latency-critical loop
where cudaMalloc/cudaFree would synchronise.  It keeps its scratch in a fixed
device array of the library.  Here it is called through the C ABI twice in a
row, on different inputs, and each result must equal the allocating
si_indexer_materialize's on the same inputs, and the oracle's where the inputs
are integer-valued (exact in fp32).  This file runs alone in a fresh process as
well as after the other tests: nothing here depends on state they leave."""

import numpy as np
import pytest
import torch

import oracle
import synth
import streaming_top_b200 as si

pytestmark = pytest.mark.gpu


def _inputs(S, T, seed, kind):
    H, D = 64, 128
    if kind == "int":
        q = synth.matrix(S * H, D, seed, synth.TENSOR_Q, "int").reshape(1, S, H, D)
        kc = synth.matrix(T, D, seed, synth.TENSOR_KC, "int").reshape(1, T, D)
        w = synth.weights(S * H, seed, synth.TENSOR_W, "pow2").reshape(1, S, H)
    else:
        sig = 1 / np.sqrt(D)
        q = synth.matrix(S * H, D, seed, synth.TENSOR_Q, "gauss", sig).reshape(1, S, H, D)
        kc = synth.matrix(T, D, seed, synth.TENSOR_KC, "gauss", sig).reshape(1, T, D)
        w = synth.weights(S * H, seed, synth.TENSOR_W, "uniform", 0.125).reshape(1, S, H)
    return {"q": q, "kc": kc, "w": w}


def _dev(inp):
    q = torch.from_numpy(inp["q"].view(np.int16)).view(torch.bfloat16).cuda()
    kc = torch.from_numpy(inp["kc"].view(np.int16)).view(torch.bfloat16).cuda()
    return q, kc, torch.from_numpy(inp["w"]).cuda()


def _call_noalloc(q, kc, w, m, k):
    """Straight through the C ABI with preallocated outputs."""
    B, S, H, D = q.shape
    T = kc.shape[1]
    idx = torch.empty((B, S, k), dtype=torch.int32, device="cuda")
    sc = torch.empty((B, S, k), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    st = si.lib().si_indexer_materialize_noalloc(q.data_ptr(), kc.data_ptr(), w.data_ptr(), B, S, T, H,
                                                 D, m, k, idx.data_ptr(), sc.data_ptr(),
                                                 torch.cuda.current_stream().cuda_stream)
    assert st == si.SI_OK, si.lib().si_last_error()
    assert si.device_status() == si.SI_OK
    return idx.cpu().numpy().reshape(-1, k), sc.cpu().numpy().reshape(-1, k)


def test_noalloc_matches_materialize_on_two_calls_in_a_row():
    cases = [(1024, 200, 4, 64, 31, "gauss"),   # ~53 MB of scratch
             (512, 128, 4, 40, 32, "int")]      # ~17 MB: the second call reuses stale contents
    for S, T, m, k, seed, kind in cases:
        inp = _inputs(S, T, seed, kind)
        q, kc, w = _dev(inp)
        gi, gs = _call_noalloc(q, kc, w, m, k)
        ri, rs = si.indexer_materialize(q, kc, w, m, k)
        assert si.device_status() == si.SI_OK
        assert np.array_equal(gi, ri.cpu().numpy().reshape(-1, k)), (S, T, kind)
        assert np.array_equal(gs, rs.cpu().numpy().reshape(-1, k)), (S, T, kind)
        if kind == "int":
            oi, osc, _ = oracle.topk(inp["q"], inp["kc"], inp["w"], m, k)
            assert np.array_equal(gi, oi) and np.array_equal(gs, osc)


def test_noalloc_rejects_problems_beyond_its_array():
    S, T, H, D, k = 1024, 1024, 64, 128, 16  # needs 4*1024*1024*65 + 256 bytes > 64 MiB
    q = torch.zeros((1, S, H, D), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((1, T, D), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((1, S, H), dtype=torch.float32, device="cuda")
    idx = torch.empty((1, S, k), dtype=torch.int32, device="cuda")
    st = si.lib().si_indexer_materialize_noalloc(q.data_ptr(), kc.data_ptr(), w.data_ptr(), 1, S, T, H, D,
                                                 4, k, idx.data_ptr(), None,
                                                 torch.cuda.current_stream().cuda_stream)
    assert st == si.SI_ERR_UNSUPPORTED
    assert b"scratch" in si.lib().si_last_error()
    assert si.device_status() == si.SI_OK
