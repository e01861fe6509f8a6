"""MXFP4 indexer keys (OCP Microscaling FP4: E2M1 codes, E8M0 scale per 32
values; queries bf16) through the C ABI on a B200, against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity

pytestmark = pytest.mark.gpu

import streaming_top_b200 as si  # noqa: E402  (fails loudly when the library is missing)


def _bf16(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def _mx_int_inputs(B, S, T, seed, H=64, D=128):
    """Integer-valued queries and MXFP4 keys whose values are multiples of
    1/4 up to 12 (scales 2^-1 .. 2^1): every logit, head sum and score is
    exact in fp32 whatever the summation order, so results are bit-exact."""
    rng = np.random.default_rng(seed)
    q = synth.f32_to_bf16_bits(rng.integers(-3, 4, size=(B, S, H, D)).astype(np.float32))
    codes = rng.integers(0, 16, size=(B, T, D)).astype(np.uint8)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    scales = rng.integers(126, 129, size=(B, T, D // 32)).astype(np.uint8)
    w = np.ldexp(1.0, -rng.integers(0, 7, size=(B, S, H))).astype(np.float32)
    return {"q": q, "kc": packed, "kc_mx_scale": scales, "w": w}


def _run(inp, m, k, **kw):
    q = _bf16(inp["q"])
    kc = torch.from_numpy(inp["kc"]).cuda()
    ms = torch.from_numpy(inp["kc_mx_scale"]).cuda()
    w = torch.from_numpy(inp["w"]).cuda()
    idx, sc = si.indexer_topk(q, kc, w, m, k, kc_mx_scale=ms, **kw)
    assert si.device_status() == si.SI_OK
    B, S = q.shape[:2]
    return idx.cpu().numpy().reshape(B * S, k), sc.cpu().numpy().reshape(B * S, k)


def test_decode_matches_oracle_bit_for_bit():
    rng = np.random.default_rng(3)
    rows, D = 4096, 128
    codes = rng.integers(0, 256, size=(rows, D // 2)).astype(np.uint8)
    scales = rng.integers(0, 253, size=(rows, D // 32)).astype(np.uint8)  # the exact range
    scales[:8] = np.array([0, 1, 2, 126, 127, 128, 251, 252], dtype=np.uint8)[:, None]
    got = si.mxfp4_to_bf16(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda())
    g = got.float().cpu().numpy().astype(np.float64)
    want = oracle.mxfp4_decode(codes, scales)
    assert np.array_equal(g, want)
    assert np.array_equal(np.signbit(g), np.signbit(want))


@pytest.mark.parametrize("B,S,T,m,k", [
    (1, 2048, 512, 4, 100),    # several key tiles and partitions
    (2, 1030, 256, 4, 64),     # two sequences, ragged query tail
    (1, 1024, 256, 4, 512),    # k > visible keys for most rows
])
def test_integer_mxfp4_bit_exact(B, S, T, m, k):
    inp = _mx_int_inputs(B, S, T, seed=S + k)
    gi, gs = _run(inp, m, k)
    oi, osc, _ = oracle.topk(inp["q"], inp["kc"], inp["w"], m, k, kc_mx_scale=inp["kc_mx_scale"])
    rows = np.arange(B * S)
    parity.check_structure(gi, gs, rows, S, T, m)
    parity.compare_exact(gi, gs, oi, osc, rows)


def test_mxfp4_row_range_and_caller_workspace():
    """The row-range entry point with MXFP4 keys and a caller-supplied
    workspace gives the whole-sequence rows."""
    B, S, T, m, k = 1, 2048, 512, 4, 96
    inp = _mx_int_inputs(B, S, T, seed=9)
    gi, gs = _run(inp, m, k)
    q, w = _bf16(inp["q"]), torch.from_numpy(inp["w"]).cuda()
    kc, ms = torch.from_numpy(inp["kc"]).cuda(), torch.from_numpy(inp["kc_mx_scale"]).cuda()
    o = si.Options()
    o.dtype = si.SI_DTYPE_MXFP4_KEYS
    need = si.lib().si_indexer_workspace_size(B, S, T, 64, 128, m, k, 0, si.ctypes.byref(o))
    ws = torch.empty(need + 17, dtype=torch.uint8, device="cuda")[17:]  # an unaligned start
    parts = []
    for r0, r1 in [(0, 700), (700, 1501), (1501, 2048)]:
        ci, cs = si.indexer_topk_rows(q[:, r0:r1].contiguous(), kc, w[:, r0:r1].contiguous(), m, k, r0,
                                      kc_mx_scale=ms, workspace=ws)
        parts.append((ci, cs))
    assert si.device_status() == si.SI_OK
    ri = torch.cat([a for a, _ in parts], dim=1).cpu().numpy().reshape(-1, k)
    rs = torch.cat([b for _, b in parts], dim=1).cpu().numpy().reshape(-1, k)
    assert np.array_equal(ri, gi) and np.array_equal(rs, gs)


def test_gaussian_mxfp4_workload_rows():
    """Planted Gaussian keys quantised to MXFP4 (the v4flash recipe at
    S=16384): sampled rows against the oracle within the float tolerance."""
    wl = synth.WORKLOADS["v4flash"]
    S = 16384
    inp = synth.make_inputs(wl, fmt="mxfp4", S=S)
    gi, gs = _run(inp, wl.m, wl.k)
    rows = np.unique(np.concatenate([synth.sample_rows(126, wl.m - 1, S, seed=5), [wl.m * wl.k - 1, S - 1]]))
    oi, _, osc64 = oracle.topk(inp["q"], inp["kc"], inp["w"], wl.m, wl.k, rows=rows,
                               kc_mx_scale=inp["kc_mx_scale"])
    parity.check_structure(gi[rows], gs[rows], rows, S, S // wl.m, wl.m)

    def full(r):
        ii, _, s64 = oracle.topk(inp["q"], inp["kc"], inp["w"], wl.m, S // wl.m, rows=[r],
                                 kc_mx_scale=inp["kc_mx_scale"])
        f = np.full(S // wl.m, np.nan)
        v = ii[0] >= 0
        f[ii[0][v]] = s64[0][v]
        return f

    st = parity.compare_tolerant(gi[rows], gs[rows], oi, osc64, rows, full)
    parity.report("workload_recall", "v4flash_mxfp4_S16384", {"stream_vs_oracle": st})
    parity.assert_recall((st, "v4flash MXFP4 keys stream vs oracle"))
