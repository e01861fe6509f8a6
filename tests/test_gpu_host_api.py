"""The host-buffer entry point si_indexer_topk_host through the binding: the
chunked, copy-overlapped path returns exactly what the device-pointer entry
points return, for every input format, ragged chunks, row ranges, page-locked
or pageable buffers and a caller workspace."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

import streaming_top_b200 as si  # noqa: E402


def _int_host(B, S, T, seed, H=64, D=128):
    q = synth.matrix(B * S * H, D, seed, synth.TENSOR_Q, "int").reshape(B, S, H, D)
    kc = synth.matrix(B * T, D, seed, synth.TENSOR_KC, "int").reshape(B, T, D)
    w = synth.weights(B * S * H, seed, synth.TENSOR_W, "pow2").reshape(B, S, H)
    return (torch.from_numpy(q.view(np.int16)).view(torch.bfloat16), torch.from_numpy(kc.view(np.int16)).view(
        torch.bfloat16), torch.from_numpy(w))


@pytest.mark.parametrize("B,S,T,k,chunk,pinned", [
    (1, 4096, 1024, 256, 1024, True),   # four chunks through two slots
    (2, 1030, 256, 96, 200, True),      # ragged last chunk, two sequences
    (1, 2048, 512, 64, 0, False),       # pageable buffers, default chunk
])
def test_host_call_equals_the_device_call(B, S, T, k, chunk, pinned):
    q, kc, w = _int_host(B, S, T, seed=71 + S)
    if pinned:
        q, kc, w = q.pin_memory(), kc.pin_memory(), w.pin_memory()
    hi, hs = si.indexer_topk_host(q, kc, w, 4, k, query_chunk=chunk)
    di, ds = si.indexer_topk(q.cuda(), kc.cuda(), w.cuda(), 4, k)
    assert torch.equal(hi, di.cpu()) and torch.equal(hs, ds.cpu())


def test_host_call_row_range_and_workspace():
    B, S, T, k, r0 = 1, 3000, 1024, 128, 1212
    q, kc, w = _int_host(B, S, T, seed=72)
    need = si.indexer_topk_host_workspace_size(B, S - r0, T, 64, 128, k, query_chunk=512)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    hq, hw = q[:, r0:].contiguous().pin_memory(), w[:, r0:].contiguous().pin_memory()
    hi, hs = si.indexer_topk_host(hq, kc.pin_memory(), hw, 4, k, row0=r0, query_chunk=512, workspace=ws)
    di, ds = si.indexer_topk(q.cuda(), kc.cuda(), w.cuda(), 4, k)
    assert torch.equal(hi, di[:, r0:].cpu()) and torch.equal(hs, ds[:, r0:].cpu())


def test_host_call_fp8_and_mxfp4_keys():
    wl = synth.WORKLOADS["tiny"]
    inp = synth.make_inputs(wl, fmt="e4m3")
    q, kc = torch.from_numpy(inp["q"]), torch.from_numpy(inp["kc"])
    w, qs, ks = (torch.from_numpy(inp[n]) for n in ("w", "q_scale", "kc_scale"))
    hi, hs = si.indexer_topk_host(q, kc, w, wl.m, wl.k, q_scale=qs, kc_scale=ks, query_chunk=256)
    di, ds = si.indexer_topk(q.cuda(), kc.cuda(), w.cuda(), wl.m, wl.k, q_scale=qs.cuda(), kc_scale=ks.cuda())
    assert torch.equal(hi, di.cpu()) and torch.equal(hs, ds.cpu())
    inp = synth.make_inputs(wl, fmt="mxfp4")
    q = torch.from_numpy(inp["q"].view(np.int16)).view(torch.bfloat16)
    kc, w, ms = (torch.from_numpy(inp[n]) for n in ("kc", "w", "kc_mx_scale"))
    hi, hs = si.indexer_topk_host(q, kc, w, wl.m, wl.k, kc_mx_scale=ms, query_chunk=300)
    di, ds = si.indexer_topk(q.cuda(), kc.cuda(), w.cuda(), wl.m, wl.k, kc_mx_scale=ms.cuda())
    assert torch.equal(hi, di.cpu()) and torch.equal(hs, ds.cpu())


def test_host_call_allocation_failure():
    q, kc, w = _int_host(1, 512, 128, seed=73)
    si.test_fail_allocations(1)
    try:
        with pytest.raises(si.SIError) as e:
            si.indexer_topk_host(q, kc, w, 4, 32)
        assert e.value.status == si.SI_ERR_OUT_OF_MEMORY
    finally:
        si.test_fail_allocations(0)
    hi, _ = si.indexer_topk_host(q, kc, w, 4, 32)
    di, _ = si.indexer_topk(q.cuda(), kc.cuda(), w.cuda(), 4, 32)
    assert torch.equal(hi, di.cpu())
