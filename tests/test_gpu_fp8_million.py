"""fp8 e4m3 scoring and the million-token workload: parity of the CUDA
streaming top-k with the CPU oracle, through the C ABI, on a B200."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity

pytestmark = pytest.mark.gpu

import streaming_top_b200 as si  # noqa: E402  (fails loudly when the library is missing)


def _e4m3_codes(vals: np.ndarray) -> np.ndarray:
    """e4m3 codes of small integers (exact in e4m3), via the input generator's encoder."""
    lut = {int(v): synth.lib().synth_f32_to_e4m3(float(v)) for v in np.unique(vals)}
    out = np.empty(vals.shape, np.uint8)
    for v, c in lut.items():
        out[vals == v] = c
    return out


def _fp8_dev(inp):
    q = torch.from_numpy(inp["q"]).cuda()
    kc = torch.from_numpy(inp["kc"]).cuda()
    w = torch.from_numpy(inp["w"]).cuda()
    qs = torch.from_numpy(inp["q_scale"]).cuda()
    ks = torch.from_numpy(inp["kc_scale"]).cuda()
    return q, kc, w, qs, ks


def _run_fp8(inp, m, k, **kw):
    q, kc, w, qs, ks = _fp8_dev(inp)
    idx, sc = si.indexer_topk(q, kc, w, m, k, q_scale=qs, kc_scale=ks, **kw)
    assert si.device_status() == si.SI_OK
    return idx.cpu().numpy().reshape(-1, k), sc.cpu().numpy().reshape(-1, k)


def _int_fp8_inputs(B, S, T, seed, H=64, D=128):
    """Integer values in {-3..3} as e4m3 codes, q scales in {1, 1/2}, kc scales
    in {1/4, 1, 2}, w = 2^-j: every product and sum is exact in fp32 (the
    weighted sum is a multiple of 2^-7 below 2^17), so any evaluation order
    gives the oracle's value."""
    # the integer generator stores bf16 bit patterns of -3..3: decode them
    qv = synth.bf16_bits_to_f32(synth.matrix(B * S * H, D, seed, synth.TENSOR_Q, "int")).astype(np.int64)
    kv = synth.bf16_bits_to_f32(synth.matrix(B * T, D, seed, synth.TENSOR_KC, "int")).astype(np.int64)
    rng = np.random.default_rng(seed)
    return {
        "q": _e4m3_codes(qv).reshape(B, S, H, D),
        "kc": _e4m3_codes(kv).reshape(B, T, D),
        "w": synth.weights(B * S * H, seed, synth.TENSOR_W, "pow2").reshape(B, S, H),
        "q_scale": rng.choice(np.float32([1.0, 0.5]), size=(B, S, H)),
        "kc_scale": rng.choice(np.float32([0.25, 1.0, 2.0]), size=(B, T)),
    }


@pytest.mark.parametrize("B,S,T,m,k,kw", [
    (1, 1024, 256, 4, 64, {}),
    (1, 2048, 512, 4, 512, {"key_tile": 128}),
    (2, 515, 128, 4, 37, {}),                       # two sequences, ragged tail
    (1, 1024, 256, 4, 64, {"key_tile": 64, "query_chunk": 256}),
])
def test_fp8_integer_inputs_bit_exact(B, S, T, m, k, kw):
    inp = _int_fp8_inputs(B, S, T, seed=21 + S)
    gi, gs = _run_fp8(inp, m, k, **kw)
    rows = np.arange(B * S)
    oi, osc, _ = oracle.topk(inp["q"], inp["kc"], inp["w"], m, k,
                             q_scale=inp["q_scale"], kc_scale=inp["kc_scale"])
    parity.check_structure(gi, gs, rows, S, T, m)
    parity.compare_exact(gi, gs, oi, osc, rows)


def _row_scores_fp8(inp, m, r, T):
    ii, _, s64 = oracle.topk(inp["q"], inp["kc"], inp["w"], m, T, rows=[r],
                             q_scale=inp["q_scale"], kc_scale=inp["kc_scale"])
    full = np.full(T, np.nan)
    v = ii[0] >= 0
    full[ii[0][v]] = s64[0][v]
    return full


def test_fp8_tiny_gaussian_workload():
    """S=1024 Gaussian inputs quantised to e4m3 with per-row scales; every row
    against the oracle on the dequantised values."""
    wl = synth.WORKLOADS["tiny"]
    inp = synth.make_inputs(wl, fmt="e4m3")
    gi, gs = _run_fp8(inp, wl.m, wl.k)
    rows = np.arange(wl.S)
    oi, _, osc64 = oracle.topk(inp["q"], inp["kc"], inp["w"], wl.m, wl.k,
                               q_scale=inp["q_scale"], kc_scale=inp["kc_scale"])
    parity.check_structure(gi, gs, rows, wl.S, wl.T, wl.m)
    st = parity.compare_tolerant(gi, gs, oi, osc64, rows, lambda r: _row_scores_fp8(inp, wl.m, r, wl.T))
    parity.report("workload_recall", "tiny_e4m3", {"stream_vs_oracle": st})
    parity.assert_recall((st, "tiny e4m3 stream vs oracle"))


def test_fp8_v4flash_sampled_rows():
    """S=65536 planted inputs in e4m3: 256 sampled rows against the oracle."""
    wl = synth.WORKLOADS["v4flash"]
    inp = synth.make_inputs(wl, fmt="e4m3")
    gi, gs = _run_fp8(inp, wl.m, wl.k)
    rows = _sample(wl)
    oi, _, osc64 = parity.oracle_rows(wl.name, rows, wl.k, fmt="e4m3", sparse=True)
    parity.check_structure(gi[rows], gs[rows], rows, wl.S, wl.T, wl.m)
    st = parity.compare_tolerant(gi[rows], gs[rows], oi, osc64, rows,
                                 lambda r: _row_scores_fp8(inp, wl.m, r, wl.T))
    parity.report("workload_recall", "v4flash_e4m3", {"stream_vs_oracle": st})
    parity.assert_recall((st, "v4flash e4m3 stream vs oracle"))


# ------------------------------------------------------ million-token workload
def _sample(wl, n=254):
    rows = synth.sample_rows(n, wl.m - 1, wl.S, seed=wl.seed)
    first_full = wl.m * wl.k - 1  # first row that sees k keys
    return np.unique(np.concatenate([rows, [first_full, wl.S - 1]])).astype(np.int64)


def _million_on_device(wl, fmt, chunk=8192):
    """The workload's inputs on the GPU, q generated and copied in chunks of
    `chunk` queries through one pinned buffer (the whole bf16 q is 16 GiB)."""
    rest = synth.make_inputs(wl, fmt=fmt, skip_q=True)
    B, S, H, D = wl.B, wl.S, wl.H, wl.D
    hdt = torch.int16 if fmt == "bf16" else torch.uint8
    ndt = np.uint16 if fmt == "bf16" else np.uint8
    q = torch.empty((B, S, H, D), dtype=hdt, device="cuda")
    qs = torch.empty((B, S, H), dtype=torch.float32, device="cuda") if fmt != "bf16" else None
    host = torch.empty((chunk, H, D), dtype=hdt).pin_memory()
    hsc = torch.empty((chunk, H), dtype=torch.float32).pin_memory()
    hnp = host.numpy().view(ndt)
    for b in range(B):
        for t0 in range(0, S, chunk):
            n = min(chunk, S - t0)
            torch.cuda.current_stream().synchronize()  # the pinned buffer is free again
            if fmt == "bf16":
                synth.q_rows(wl, b, t0, n, fmt, out=hnp[:n])
            else:
                synth.q_rows(wl, b, t0, n, fmt, out=hnp[:n], scale_out=hsc.numpy()[:n])
                qs[b, t0:t0 + n].copy_(hsc[:n], non_blocking=True)
            q[b, t0:t0 + n].copy_(host[:n], non_blocking=True)
    torch.cuda.synchronize()
    if fmt == "bf16":
        kc = torch.from_numpy(rest["kc"].view(np.int16)).view(torch.bfloat16).cuda()
        q = q.view(torch.bfloat16)
        ks = None
    else:
        kc = torch.from_numpy(rest["kc"]).cuda()
        ks = torch.from_numpy(rest["kc_scale"]).cuda()
    w = torch.from_numpy(rest["w"]).cuda()
    return q, kc, w, qs, ks


@pytest.mark.slow
@pytest.mark.parametrize("fmt", ["bf16", "e4m3"])
def test_million_token_sampled_rows(fmt):
    """S=1,048,576 (T=262,144), k=512, planted inputs: the whole sequence in one
    call, 256 sampled rows against the oracle (which regenerates only those
    rows of q)."""
    wl = synth.WORKLOADS["million"]
    q, kc, w, qs, ks = _million_on_device(wl, fmt)
    idx, sc = si.indexer_topk(q, kc, w, wl.m, wl.k, q_scale=qs, kc_scale=ks)
    assert si.device_status() == si.SI_OK
    rows = _sample(wl)
    sel = torch.from_numpy(rows).cuda()
    gi = idx.view(-1, wl.k).index_select(0, sel).cpu().numpy()
    gs = sc.view(-1, wl.k).index_select(0, sel).cpu().numpy()
    del q, kc, w, qs, ks, idx, sc
    torch.cuda.empty_cache()
    oi, _, osc64 = parity.oracle_rows(wl.name, rows, wl.k, fmt=fmt, sparse=True)
    parity.check_structure(gi, gs, rows, wl.S, wl.T, wl.m)

    def row_scores(r):
        inp = synth.make_inputs_rows(wl, [r], fmt=fmt)
        if fmt == "bf16":
            return oracle.scores(inp["q"], inp["kc"], inp["w"], wl.m, r)
        return _row_scores_fp8(inp, wl.m, r, wl.T)

    st = parity.compare_tolerant(gi, gs, oi, osc64, rows, row_scores)
    parity.report("workload_recall", f"million_{fmt}", {"stream_vs_oracle": st})
    parity.assert_recall((st, f"million {fmt} stream vs oracle"))
