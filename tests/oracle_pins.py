"""Pins for the CPU oracle: checks that do not restate its formula.

Each check takes a ctypes handle on an oracle library, so the same checks run
on the real oracle (test_oracle_pins.py) and on copies with a planted mistake
(test_oracle_mutants.py), which must each fail at least one of them.

What pins what:
  hand_cases        -- values worked out on paper (tests/golden/hand_cases.json)
  onehot_matmul     -- one head selected: scores reduce to ReLU(K @ q), a
                       numpy matmul; selection to numpy's stable argsort
  positive_closed   -- all logits positive: ReLU is the identity, so the
                       score is K @ (Q^T w), a numpy matmul
  visible_closed    -- the count of returned keys with k >= T equals the
                       closed form sum_t min(T, floor((t+1)/m))
  causal            -- no returned key ends after its query
  prefix            -- top-k is a prefix of top-(k+1)
  brute_subsets     -- the returned set is the unique k-subset whose every
                       member beats every non-member, found by enumeration
  invariances       -- permuting heads (q and w together), scaling w by 2^j,
                       w = 0 (all ties) -> indices 0..n-1
  batch_independent -- sequence b's result does not depend on other sequences
  fp8_matches_bf16  -- e4m3 inputs whose values are bf16-exact give the bf16 result
"""
from __future__ import annotations

import itertools
import json
import os

import numpy as np

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _bits(x) -> np.ndarray:
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _f(bits) -> np.ndarray:
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def _int_problem(rng, B, S, T, H, D, lo=-3, hi=3):
    q = _bits(rng.integers(lo, hi + 1, size=(B, S, H, D)))
    kc = _bits(rng.integers(lo, hi + 1, size=(B, T, D)))
    w = np.ldexp(1.0, -rng.integers(0, 7, size=(B, S, H))).astype(np.float32)
    return q, kc, w


def hand_cases(lib):
    data = json.load(open(os.path.join(GOLDEN, "hand_cases.json")))
    for case in data["cases"]:
        B, S, T, H, D, m, k = (case[x] for x in ("B", "S", "T", "H", "D", "m", "k"))
        q = np.zeros((B * S, H, D), dtype=np.float32)
        w = np.zeros((B * S, H), dtype=np.float32)
        for r, v in case["q"].items():
            q[int(r)] = np.asarray(v, dtype=np.float32)
        for r, v in case["w"].items():
            w[int(r)] = np.asarray(v, dtype=np.float32)
        kc = np.asarray(case["kc"], dtype=np.float32).reshape(B, T, D)
        rows = np.array(sorted(int(r) for r in case["expect"]), dtype=np.int64)
        idx, sc, _ = oracle.topk(_bits(q).reshape(B, S, H, D), _bits(kc), w.reshape(B, S, H), m, k,
                                 rows=rows, lib=lib)
        for i, r in enumerate(rows):
            e = case["expect"][str(r)]
            want_idx = np.asarray(e["idx"], dtype=np.int32)
            want_sc = np.asarray([float(x) for x in e["score"]], dtype=np.float32)
            assert np.array_equal(idx[i], want_idx), (case["name"], r, idx[i], want_idx)
            assert np.array_equal(sc[i], want_sc), (case["name"], r, sc[i], want_sc)


def onehot_matmul(lib, seed=11):
    rng = np.random.default_rng(seed)
    B, S, T, H, D, m, k = 1, 48, 12, 4, 8, 4, 5
    q, kc, _ = _int_problem(rng, B, S, T, H, D)
    for h0 in range(H):
        w = np.zeros((B, S, H), dtype=np.float32)
        w[..., h0] = 1.0
        idx, sc, _ = oracle.topk(q, kc, w, m, k, lib=lib)
        K = _f(kc[0])
        for t in range(S):
            n = min(T, (t + 1) // m)
            s = np.maximum(K[:n] @ _f(q[0, t, h0]), 0.0)
            order = np.argsort(-s, kind="stable")[:k]
            want = np.full(k, -1, dtype=np.int32)
            want[: len(order)] = order
            assert np.array_equal(idx[t], want), (h0, t, idx[t], want)
            assert np.array_equal(sc[t, : len(order)], s[order].astype(np.float32))


def positive_closed(lib, seed=12):
    rng = np.random.default_rng(seed)
    B, S, T, H, D, m, k = 1, 40, 10, 3, 6, 4, 4
    q, kc, w = _int_problem(rng, B, S, T, H, D, lo=1, hi=4)
    idx, sc, sc64 = oracle.topk(q, kc, w, m, k, lib=lib)
    K = _f(kc[0])
    for t in range(S):
        n = min(T, (t + 1) // m)
        qw = _f(q[0, t]).T @ w[0, t].astype(np.float64)  # (D,)
        s = K[:n] @ qw
        order = np.argsort(-s, kind="stable")[:k]
        assert np.array_equal(idx[t, : len(order)], order), (t, idx[t], order)
        assert np.array_equal(sc64[t, : len(order)], s[order])


def visible_closed(lib):
    rng = np.random.default_rng(13)
    for (S, T, m) in [(32, 8, 4), (30, 8, 4), (24, 5, 3), (17, 16, 1), (20, 4, 2)]:
        H, D = 2, 4
        q, kc, w = _int_problem(rng, 1, S, T, H, D)
        idx, _, _ = oracle.topk(q, kc, w, m, T, lib=lib)
        assert int((idx >= 0).sum()) == synth.visible_pairs(S, T, m), (S, T, m)
        if S == m * T:
            assert int((idx >= 0).sum()) == m * T * (T - 1) // 2 + T


def causal(lib):
    rng = np.random.default_rng(14)
    S, T, m, k = 64, 16, 4, 6
    q, kc, w = _int_problem(rng, 1, S, T, 2, 4)
    idx, sc, _ = oracle.topk(q, kc, w, m, k, lib=lib)
    for t in range(S):
        valid = idx[t][idx[t] >= 0]
        assert all(s * m + m - 1 <= t for s in valid), (t, valid)
        n = min(T, (t + 1) // m)
        assert len(valid) == min(k, n)
        assert len(set(valid.tolist())) == len(valid)
        assert np.all(np.isneginf(sc[t][idx[t] < 0]))


def prefix(lib):
    rng = np.random.default_rng(15)
    S, T, m = 48, 12, 4
    q, kc, w = _int_problem(rng, 1, S, T, 3, 5)
    prev = None
    for k in range(1, T + 2):
        idx, _, _ = oracle.topk(q, kc, w, m, k, lib=lib)
        if prev is not None:
            assert np.array_equal(idx[:, : k - 1], prev), k
        prev = idx


def brute_subsets(lib):
    rng = np.random.default_rng(16)
    S, T, m = 36, 9, 4
    q, kc, w = _int_problem(rng, 1, S, T, 2, 3, lo=-2, hi=2)
    for t in (11, 23, 35):
        n = min(T, (t + 1) // m)
        sc = oracle.scores(q, kc, w, m, t, lib=lib)[:n]
        key = [(sc[s], -s) for s in range(n)]
        for k in range(1, n + 1):
            idx, _, _ = oracle.topk(q, kc, w, m, k, rows=[t], lib=lib)
            winners = [A for A in itertools.combinations(range(n), k)
                       if min(key[a] for a in A) > max((key[b] for b in range(n) if b not in A),
                                                       default=(-np.inf, -np.inf))]
            assert len(winners) == 1
            want = sorted(winners[0], key=lambda s: (-sc[s], s))
            assert idx[0].tolist() == want, (t, k, idx[0], want)


def invariances(lib):
    rng = np.random.default_rng(17)
    S, T, H, D, m, k = 40, 10, 4, 6, 4, 5
    q, kc, w = _int_problem(rng, 1, S, T, H, D)
    idx, sc, _ = oracle.topk(q, kc, w, m, k, lib=lib)
    perm = rng.permutation(H)
    idx2, sc2, _ = oracle.topk(np.ascontiguousarray(q[:, :, perm]), kc,
                               np.ascontiguousarray(w[:, :, perm]), m, k, lib=lib)
    assert np.array_equal(idx, idx2) and np.array_equal(sc, sc2)
    for j in (-3, 2):
        idx3, sc3, _ = oracle.topk(q, kc, (w * np.float32(2.0 ** j)).astype(np.float32), m, k, lib=lib)
        assert np.array_equal(idx, idx3)
        v = idx >= 0
        assert np.array_equal(sc3[v], sc[v] * np.float32(2.0 ** j))
    idx4, sc4, _ = oracle.topk(q, kc, np.zeros_like(w), m, k, lib=lib)
    for t in range(S):
        n = min(T, (t + 1) // m)
        want = np.full(k, -1, dtype=np.int32)
        want[: min(k, n)] = np.arange(min(k, n))
        assert np.array_equal(idx4[t], want)
        assert np.all(sc4[t, : min(k, n)] == 0.0)


def batch_independent(lib):
    rng = np.random.default_rng(18)
    B, S, T, H, D, m, k = 3, 24, 6, 2, 4, 4, 4
    q, kc, w = _int_problem(rng, B, S, T, H, D)
    idx, sc, _ = oracle.topk(q, kc, w, m, k, lib=lib)
    for b in range(B):
        i1, s1, _ = oracle.topk(np.ascontiguousarray(q[b:b + 1]), np.ascontiguousarray(kc[b:b + 1]),
                                np.ascontiguousarray(w[b:b + 1]), m, k, lib=lib)
        assert np.array_equal(idx[b * S:(b + 1) * S], i1), b
        assert np.array_equal(sc[b * S:(b + 1) * S], s1), b
    # a different sequence's keys give a different answer somewhere
    i_sw, _, _ = oracle.topk(q, np.ascontiguousarray(kc[::-1]), w, m, k, lib=lib)
    assert not np.array_equal(i_sw, idx)


def fp8_matches_bf16(lib):
    rng = np.random.default_rng(19)
    B, S, T, H, D, m, k = 1, 32, 8, 3, 16, 4, 5
    q8 = rng.integers(0, 256, size=(B, S, H, D)).astype(np.uint8)
    kc8 = rng.integers(0, 256, size=(B, T, D)).astype(np.uint8)
    q8[(q8 & 0x7F) == 0x7F] = 0x10   # no NaN codes
    kc8[(kc8 & 0x7F) == 0x7F] = 0x10
    q_scale = np.ldexp(1.0, rng.integers(-2, 3, size=(B, S, H))).astype(np.float32)
    kc_scale = np.ldexp(1.0, rng.integers(-2, 3, size=(B, T))).astype(np.float32)
    w = rng.random((B, S, H)).astype(np.float32)
    import torch
    qv = torch.from_numpy(q8).view(torch.float8_e4m3fn).float().numpy() * q_scale[..., None]
    kv = torch.from_numpy(kc8).view(torch.float8_e4m3fn).float().numpy() * kc_scale[..., None]
    qb, kb = _bits(qv), _bits(kv)
    assert np.array_equal(_f(qb), qv.astype(np.float64))  # e4m3 * 2^j is bf16-exact
    i8, s8, _ = oracle.topk(q8, kc8, w, m, k, q_scale=q_scale, kc_scale=kc_scale, lib=lib)
    ib, sb, _ = oracle.topk(qb, kb, w, m, k, lib=lib)
    assert np.array_equal(i8, ib) and np.array_equal(s8, sb)


def mxfp4_matches_bf16(lib):
    """MXFP4 keys (OCP Microscaling FP4) against the bf16 path on the same
    values.  The codes are decoded here by ml_dtypes' float4_e2m1fn (a
    library conversion, not the oracle's bit arithmetic) times 2^(scale-127)
    per 32-value block, value d in the low nibble of byte d/2 when d is even;
    such keys are exact in bf16, so both oracle paths must agree bit for
    bit, and the oracle's own decode must give the same values."""
    import ml_dtypes
    rng = np.random.default_rng(23)
    B, S, T, H, D, m, k = 2, 40, 10, 3, 64, 4, 6
    codes = rng.integers(0, 16, size=(B, T, D)).astype(np.uint8)
    scales = rng.integers(118, 136, size=(B, T, D // 32)).astype(np.uint8)
    step = np.ldexp(1.0, scales.astype(np.int64) - 127).repeat(32, axis=-1)
    vals = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64) * step
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    kb = _bits(vals)
    assert np.array_equal(_f(kb), vals)  # E2M1 times a power of two is bf16-exact here
    assert np.array_equal(oracle.mxfp4_decode(packed, scales, lib=lib), vals)
    q = _bits(rng.standard_normal((B, S, H, D)) / 8)
    w = rng.random((B, S, H)).astype(np.float32)
    imx, smx, _ = oracle.topk(q, packed, w, m, k, kc_mx_scale=scales, lib=lib)
    ib, sb, _ = oracle.topk(q, kb, w, m, k, lib=lib)
    assert np.array_equal(imx, ib) and np.array_equal(smx, sb)
    assert np.any(imx[:, 0] > 0)  # the keys are not all tied


def two_stage_hand_case(lib):
    """The two-stage case worked by hand in tests/golden/two_stage_hand.json."""
    c = json.load(open(os.path.join(GOLDEN, "two_stage_hand.json")))
    S, T, H, D = c["S"], c["T"], c["H"], c["D"]
    q = _bits(np.array(c["q"], dtype=np.float32).reshape(1, S, H, D))
    kc = _bits(np.array(c["kc"], dtype=np.float32).reshape(1, T, D))
    w = np.array(c["w"], dtype=np.float32).reshape(1, S, H)
    idx, sc, _ = oracle.topk_two_stage(q, kc, w, c["m"], c["k"], G=c["block"], n_keep=c["n_keep"], lib=lib)
    want = np.array([[float(x) for x in r] for r in c["score"]], dtype=np.float32)
    assert np.array_equal(idx, np.array(c["idx"], dtype=np.int32)), idx
    assert np.array_equal(sc, want), sc


def two_stage_all_kept(lib):
    """With at most n_keep complete visible blocks every visible key is a
    candidate, so the two-stage result is the one-stage top-k (rows with an
    incomplete last block included: S is not a multiple of m*G)."""
    rng = np.random.default_rng(29)
    B, S, T, H, D, m, k, G = 2, 300, 72, 3, 16, 4, 10, 8
    q = _bits(rng.standard_normal((B, S, H, D)))
    kc = _bits(rng.standard_normal((B, T, D)))
    w = rng.random((B, S, H)).astype(np.float32)
    i1, s1, _ = oracle.topk(q, kc, w, m, k, lib=lib)
    for keep in (T // G, T // G + 5):
        i2, s2, _ = oracle.topk_two_stage(q, kc, w, m, k, G=G, n_keep=keep, lib=lib)
        assert np.array_equal(i1, i2) and np.array_equal(s1, s2), keep


def two_stage_one_key_per_block(lib):
    """Blocks with a single nonzero key (at a random position) and positive
    values: a block's pooled key is that key / G exactly, its coarse score is
    that key's score / G, so the kept blocks are those holding the n_keep best
    keys and the two-stage top-n_keep equals the one-stage top-n_keep."""
    rng = np.random.default_rng(31)
    B, S, T, H, D, m, G, keep = 1, 400, 100, 2, 8, 4, 8, 5
    q = _bits(rng.random((B, S, H, D)) + 0.25)
    kc = np.zeros((B, T, D), dtype=np.float32)
    pos = rng.integers(0, G, size=(B, (T + G - 1) // G))
    for j in range(pos.shape[1]):
        s = j * G + pos[0, j]
        if s < T:
            kc[0, s] = rng.random(D) + 0.25
    kc = _bits(kc)
    w = (rng.random((B, S, H)) + 0.1).astype(np.float32)
    rows = np.arange(m * G * (keep + 1), S)  # rows with more than n_keep complete blocks
    i1, s1, _ = oracle.topk(q, kc, w, m, keep, rows=rows, lib=lib)
    i2, s2, _ = oracle.topk_two_stage(q, kc, w, m, keep, G=G, n_keep=keep, rows=rows, lib=lib)
    assert np.all(s1 > 0)
    assert np.array_equal(i1, i2) and np.array_equal(s1, s2)


def two_stage_pooled_keys(lib):
    """The pooled keys against numpy's block mean rounded to bf16 by
    ml_dtypes (a library conversion, round to nearest even)."""
    import ml_dtypes
    rng = np.random.default_rng(37)
    kc = _bits(rng.standard_normal((2, 70, 16)) * 3)
    got = oracle.pool_keys(kc, 8, lib=lib)
    blocks = _f(kc)[:, :64].reshape(2, 8, 8, 16)
    want = blocks.mean(axis=2).astype(ml_dtypes.bfloat16).astype(np.float64)
    assert got.shape == (2, 8, 16) and np.array_equal(got, want)


def _attn_problem(rng, B=2, S=5, T=12, H=3, Dk=16, k=6):
    q = _bits(rng.standard_normal((B, S, H, Dk)))
    kv = _bits(rng.standard_normal((B, T, Dk)))
    idx = np.stack([np.stack([rng.permutation(T)[:k] for _ in range(S)]) for _ in range(B)]).astype(np.int32)
    idx[0, 1, 4:] = -1   # padding
    idx[1, 2, :] = -1    # a row with nothing selected
    return q, kv, idx


def attn_matches_sdpa(lib):
    """Sparse attention against torch's scaled_dot_product_attention (fp64,
    CPU) over each query's gathered entries, and lse against logsumexp."""
    import torch
    rng = np.random.default_rng(41)
    q, kv, idx = _attn_problem(rng)
    Dv = 10
    out, lse = oracle.sparse_attention(q, kv, idx, Dv, lib=lib)
    Q, KV = torch.from_numpy(_f(q)), torch.from_numpy(_f(kv))
    B, S, H, Dk = q.shape
    for b in range(B):
        for t in range(S):
            sel = [int(x) for x in idx[b, t] if x >= 0]
            if not sel:
                assert np.all(out[b, t] == 0) and np.all(np.isneginf(lse[b, t]))
                continue
            K = KV[b, sel]                       # [n, Dk]
            want = torch.nn.functional.scaled_dot_product_attention(
                Q[b, t][:, None, :], K[None].expand(H, -1, -1), K[None, :, :Dv].expand(H, -1, -1))[:, 0]
            assert np.allclose(out[b, t], want.numpy(), rtol=1e-12, atol=1e-13)
            want_lse = torch.logsumexp((Q[b, t] @ K.T) / np.sqrt(Dk), dim=-1)
            assert np.allclose(lse[b, t], want_lse.numpy(), rtol=1e-12, atol=1e-13)


def attn_special_cases(lib):
    """One selected entry gives exactly its value rows (weight 1); all-zero
    queries give the plain mean of the selected values; permuting the
    selection and moving the padding changes nothing beyond rounding."""
    rng = np.random.default_rng(43)
    q, kv, idx = _attn_problem(rng)
    Dv = 16
    one = np.full_like(idx, -1)
    one[:, :, 2] = idx[:, :, 0].clip(0)
    out, lse = oracle.sparse_attention(q, kv, one, Dv, lib=lib)
    vals = _f(kv)
    for b in range(q.shape[0]):
        for t in range(q.shape[1]):
            assert np.array_equal(out[b, t], np.broadcast_to(vals[b, one[b, t, 2], :Dv], out[b, t].shape))
    zq = np.zeros_like(q)
    out0, _ = oracle.sparse_attention(zq, kv, idx, Dv, lib=lib)
    for b in range(q.shape[0]):
        for t in range(q.shape[1]):
            sel = [int(x) for x in idx[b, t] if x >= 0]
            if sel:
                assert np.allclose(out0[b, t], vals[b, sel, :Dv].mean(axis=0), rtol=1e-14, atol=1e-15)
    perm = idx[:, :, ::-1].copy()
    out_p, lse_p = oracle.sparse_attention(q, kv, perm, Dv, lib=lib)
    out_r, lse_r = oracle.sparse_attention(q, kv, idx, Dv, lib=lib)
    assert np.allclose(out_p, out_r, rtol=1e-12, atol=1e-14)
    assert np.allclose(lse_p[np.isfinite(lse_r)], lse_r[np.isfinite(lse_r)], rtol=1e-13)


ALL = [hand_cases, onehot_matmul, positive_closed, visible_closed, causal, prefix, brute_subsets,
       invariances, batch_independent, fp8_matches_bf16, mxfp4_matches_bf16, two_stage_all_kept,
       two_stage_one_key_per_block, two_stage_pooled_keys, two_stage_hand_case, attn_matches_sdpa,
       attn_special_cases]
