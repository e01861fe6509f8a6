"""Failure paths on a B200, without faulting the GPU: allocation failures
made on the host (the library's allocation-failure test hook) and a bounded
wait that runs out, reported through a call's own device status word."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity

pytestmark = pytest.mark.gpu

import streaming_top_b200 as si  # noqa: E402


def _int_dev(B, S, T, seed, H=64, D=128):
    q = synth.matrix(B * S * H, D, seed, synth.TENSOR_Q, "int").reshape(B, S, H, D)
    kc = synth.matrix(B * T, D, seed, synth.TENSOR_KC, "int").reshape(B, T, D)
    w = synth.weights(B * S * H, seed, synth.TENSOR_W, "pow2").reshape(B, S, H)
    host = {"q": q, "kc": kc, "w": w}
    dev = (torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).cuda(),
           torch.from_numpy(kc.view(np.int16)).view(torch.bfloat16).cuda(), torch.from_numpy(w).cuda())
    return host, dev


def _mxfp4_call(q, kc, w):
    codes = torch.zeros((kc.shape[0], kc.shape[1], 64), dtype=torch.uint8, device="cuda")
    scales = torch.full((kc.shape[0], kc.shape[1], 4), 127, dtype=torch.uint8, device="cuda")
    return si.indexer_topk(q, codes, w, 4, 32, kc_mx_scale=scales)


@pytest.mark.parametrize("path", ["mxfp4_keys", "materialize", "two_stage"])
def test_allocation_failure_is_reported_and_the_context_survives(path):
    """With the hook set, the call that needs scratch returns
    SI_ERR_OUT_OF_MEMORY; the hook is used up and the next call succeeds with
    the exact result."""
    host, (q, kc, w) = _int_dev(1, 512, 128, seed=51)
    calls = {
        "mxfp4_keys": lambda: _mxfp4_call(q, kc, w),
        "materialize": lambda: si.indexer_materialize(q, kc, w, 4, 32),
        "two_stage": lambda: si.indexer_topk_two_stage(q, kc, w, 4, 32, block=8, n_keep=4),
    }
    si.test_fail_allocations(1)
    try:
        with pytest.raises(si.SIError) as e:
            calls[path]()
        assert e.value.status == si.SI_ERR_OUT_OF_MEMORY
        assert b"test hook" in si.lib().si_last_error()
    finally:
        si.test_fail_allocations(0)
    assert si.device_status() == si.SI_OK
    calls[path]()  # the hook is used up: the same call now runs
    assert si.device_status() == si.SI_OK
    gi, gs = si.indexer_materialize(q, kc, w, 4, 32)
    oi, osc, _ = oracle.topk(host["q"], host["kc"], host["w"], 4, 32)
    parity.compare_exact(gi.cpu().numpy().reshape(-1, 32), gs.cpu().numpy().reshape(-1, 32), oi, osc,
                         np.arange(512))


def test_timeout_goes_to_the_calls_own_status_word():
    """A bounded wait that runs out is written to the call's device_status
    word, not to the shared per-device record; a normal call given a status
    word leaves it zero."""
    host, (q, kc, w) = _int_dev(1, 1024, 256, seed=52)
    out = torch.empty((1, 1024, 64), dtype=torch.int32, device="cuda")
    word = torch.zeros(2, dtype=torch.int32, device="cuda")
    assert si.test_stream_timeout(q, kc, w, 4, 64, out, wait_limit_ns=50_000_000, device_status=word) == si.SI_OK
    torch.cuda.synchronize()
    assert int(word[0]) == si.SI_ERR_TIMEOUT and int(word[1]) > 0
    assert si.device_status() == si.SI_OK  # the shared record was not touched
    word.zero_()
    gi, gs = si.indexer_topk(q, kc, w, 4, 64, device_status=word)
    torch.cuda.synchronize()
    assert int(word[0]) == 0 and int(word[1]) == 0
    oi, osc, _ = oracle.topk(host["q"], host["kc"], host["w"], 4, 64)
    parity.compare_exact(gi.cpu().numpy().reshape(-1, 64), gs.cpu().numpy().reshape(-1, 64), oi, osc,
                         np.arange(1024))
