"""The sparse attention over the selected latents (``si_sparse_attention``)
against the oracle (``oracle_sparse_attention_bf16``, fp64), element by
element, and its special cases.

Tolerance, from the arithmetic: the logits are fp32 sums of exact bf16
products (error ~1e-6 relative), exp and log are the fast single-precision
functions (a few ulp), and the softmax weights are rounded to bf16 (relative
error <= 2^-9 each) before the value product, which the sum of the rounded
weights normalises.  A weighted mean whose weights move by <= 2^-9 relative
moves by <= 2^-9 * max_j |v_j - out|, so |out - oracle| <= 2^-8 * max|v| plus
the bf16 rounding of the output (2^-9 |out|); lse = scale*max + ln(sum) moves
by <= 2^-9 from the rounded weights plus the fp32 errors: 4e-3 absolute."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

import streaming_top_b200 as si  # noqa: E402

H, DK, DV = 64, 576, 512


def _bf16_to_f32(bits):
    return synth.bf16_bits_to_f32(bits)


def _run(q, kv, idx, scale=0.0):
    qd = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).cuda()
    kd = torch.from_numpy(kv.view(np.int16)).view(torch.bfloat16).cuda()
    out, lse = si.sparse_attention(qd, kd, torch.from_numpy(idx).cuda(), scale=scale)
    assert si.device_status() == si.SI_OK
    return out.float().cpu().numpy(), lse.cpu().numpy()


def _check(q, kv, idx, scale=0.0):
    go, gl = _run(q, kv, idx, scale)
    ro, rl = oracle.sparse_attention(q, kv, idx, DV, scale=scale if scale > 0 else None)
    vmax = np.abs(_bf16_to_f32(kv[..., :DV])).max()
    tol = 2.0 ** -8 * vmax + 2.0 ** -9 * np.abs(ro)
    err = np.abs(go - ro)
    assert np.all(err <= tol), (float(err.max()), float((err - tol).max()))
    fin = np.isfinite(rl)
    assert np.array_equal(fin, np.isfinite(gl)) and np.all(np.isneginf(gl[~fin]))
    assert np.all(np.abs(gl[fin] - rl[fin]) <= 4e-3), float(np.abs(gl[fin] - rl[fin]).max())
    return go, gl


def _selection(B, S, T, k, seed, pad_frac=0.0):
    """Distinct random entries per row, a fraction of them replaced by -1."""
    rng = np.random.default_rng(seed)
    idx = np.stack([np.stack([rng.choice(T, size=k, replace=False) for _ in range(S)]) for _ in range(B)])
    idx = idx.astype(np.int32)
    if pad_frac:
        idx[rng.random(idx.shape) < pad_frac] = -1
    return idx


@pytest.mark.parametrize("B,S,T,k,pad", [
    (1, 160, 1024, 512, 0.0),     # more queries than SMs: a CTA takes two
    (2, 40, 700, 256, 0.1),       # two sequences, padding inside the selection
    (1, 24, 512, 128, 0.0),       # one entry tile
    (1, 16, 384, 384, 0.3),
])
def test_attention_matches_the_oracle(B, S, T, k, pad):
    q, kv = synth.attention_inputs(B, S, T, seed=100 + S)
    _check(q, kv, _selection(B, S, T, k, seed=S, pad_frac=pad))


def test_attention_over_the_indexer_selection():
    """The consumer on the indexer's own output: the top-512 of the planted
    v4flash recipe at S = 4096 (the last rows select 512 of 1024 keys), with
    the early rows padded."""
    wl = synth.WORKLOADS["v4flash"]
    S = 4096
    inp = synth.make_inputs(wl, S=S)
    qd = torch.from_numpy(inp["q"].view(np.int16)).view(torch.bfloat16).cuda()
    kd = torch.from_numpy(inp["kc"].view(np.int16)).view(torch.bfloat16).cuda()
    idx, _ = si.indexer_topk(qd, kd, torch.from_numpy(inp["w"]).cuda(), wl.m, 512)
    rows = np.r_[0:8, 2040:2048, S - 8:S]
    sel = idx.cpu().numpy()[:, rows]
    q, kv = synth.attention_inputs(1, len(rows), S // wl.m, seed=7)
    _check(q, kv, np.ascontiguousarray(sel))


def test_attention_full_size_sampled_rows():
    """The launch the bench times: 65,536 queries x 64 heads over T = 16,384
    latents, each query's selection the indexer's top-512 of the planted
    v4flash inputs (seed 3), the attention inputs drawn as the bench draws
    them.  48 sampled queries (the first, the last, and uniformly drawn ones)
    against the oracle, the rest only for finiteness."""
    wl = synth.WORKLOADS["v4flash"]
    inp = synth.make_inputs(wl)
    qi = torch.from_numpy(inp["q"].view(np.int16)).view(torch.bfloat16).cuda()
    kc = torch.from_numpy(inp["kc"].view(np.int16)).view(torch.bfloat16).cuda()
    idx, _ = si.indexer_topk(qi, kc, torch.from_numpy(inp["w"]).cuda(), wl.m, wl.k)
    del qi, kc, inp
    q, kv = synth.attention_inputs(wl.B, wl.S, wl.T, seed=wl.seed + 500)
    qd = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).cuda()
    kd = torch.from_numpy(kv.view(np.int16)).view(torch.bfloat16).cuda()
    out, lse = si.sparse_attention(qd, kd, idx)
    assert si.device_status() == si.SI_OK
    del qd, kd
    rows = np.unique(np.r_[0, 1, wl.S - 1, synth.sample_rows(45, 2, wl.S - 1, seed=11)])
    rt = torch.from_numpy(rows).cuda()
    go = out[:, rt].float().cpu().numpy()
    gl = lse[:, rt].cpu().numpy()
    sel = np.ascontiguousarray(idx[:, rt].cpu().numpy())
    ro, rl = oracle.sparse_attention(np.ascontiguousarray(q[:, rows]), kv, sel, DV)
    vmax = np.abs(_bf16_to_f32(kv[..., :DV])).max()
    err = np.abs(go - ro)
    assert np.all(err <= 2.0 ** -8 * vmax + 2.0 ** -9 * np.abs(ro)), float(err.max())
    fin = np.isfinite(rl)
    assert np.array_equal(fin, np.isfinite(gl)) and np.all(np.isneginf(gl[~fin]))
    assert np.all(np.abs(gl[fin] - rl[fin]) <= 4e-3), float(np.abs(gl[fin] - rl[fin]).max())
    # every query attends over at least one key (query t sees (t+1)//4 >= 1 keys from t = 3 on)
    assert bool(torch.isfinite(lse[:, 3:]).all())


def test_attention_special_cases():
    T, k = 256, 128
    q, kv = synth.attention_inputs(1, 4, T, seed=9)
    idx = np.full((1, 4, k), -1, np.int32)
    idx[0, 0, 37] = 11           # one entry: out is exactly that entry's value
    idx[0, 2, :] = np.arange(k)  # all entries of the first tile
    idx[0, 3, ::2] = np.arange(0, 2 * k, 4)[: k // 2]  # every other slot padded
    go, gl = _check(q, kv, idx)
    v11 = _bf16_to_f32(kv[0, 11, :DV])
    assert np.array_equal(go[0, 0], np.broadcast_to(v11, (H, DV)))
    assert np.all(go[0, 1] == 0.0) and np.all(np.isneginf(gl[0, 1]))   # nothing selected
    # a permutation of the selection (padding moved) changes nothing beyond rounding
    perm = np.random.default_rng(3).permutation(k)
    idx2 = idx.copy()
    idx2[0, 3] = idx[0, 3, perm]
    go2, gl2 = _run(q, kv, idx2)
    assert np.allclose(go2[0, 3], go[0, 3], atol=2.0 ** -8 * np.abs(_bf16_to_f32(kv)).max())
    assert np.allclose(gl2[0, 3], gl[0, 3], atol=1e-5)


def test_attention_integer_inputs_exact_where_the_weights_are():
    """Integer latents and a zero query: every logit is 0, every weight is
    exactly 1 in bf16, so the output is the exact mean of the selected values
    (rounded once to bf16) and lse = ln(count)."""
    T, k = 300, 256
    q, kv = synth.attention_inputs(1, 8, T, seed=12, kind="int")
    q[:] = 0
    idx = _selection(1, 8, T, k, seed=4, pad_frac=0.25)
    go, gl = _run(q, kv, idx)
    vals = _bf16_to_f32(kv[0])
    for t in range(8):
        sel = idx[0, t][idx[0, t] >= 0]
        mean = vals[sel, :DV].astype(np.float64).mean(axis=0)
        want = _bf16_to_f32(synth.f32_to_bf16_bits(mean.astype(np.float32)))
        assert np.allclose(go[0, t], np.broadcast_to(want, (H, DV)), rtol=0, atol=2.0 ** -8 * np.abs(mean).max() + 1e-6)
        assert np.allclose(gl[0, t], np.log(len(sel)), atol=1e-5)


def test_attention_refuses_other_shapes():
    q = torch.zeros((1, 4, 64, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((1, 16, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((1, 4, 128), dtype=torch.int32, device="cuda")
    with pytest.raises(si.SIError) as e:
        si.sparse_attention(q, kv, idx)
    assert e.value.status == si.SI_ERR_UNSUPPORTED
