"""Parity of the CUDA streaming top-k (and the in-library materialize path)
with the CPU oracle, through the C ABI, on a B200."""
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
    w = torch.from_numpy(inp["w"]).cuda()
    return q, kc, w


def _run(inp, m, k, **kw):
    q, kc, w = _dev(inp)
    idx, sc = si.indexer_topk(q, kc, w, m, k, **kw)
    assert si.device_status() == si.SI_OK
    return idx.cpu().numpy().reshape(-1, k), sc.cpu().numpy().reshape(-1, k)


def _mat(inp, m, k):
    q, kc, w = _dev(inp)
    idx, sc = si.indexer_materialize(q, kc, w, m, k)
    assert si.device_status() == si.SI_OK
    return idx.cpu().numpy().reshape(-1, k), sc.cpu().numpy().reshape(-1, k)


def _int_inputs(B, S, T, seed, H=64, D=128):
    q = synth.matrix(B * S * H, D, seed, synth.TENSOR_Q, "int").reshape(B, S, H, D)
    kc = synth.matrix(B * T, D, seed, synth.TENSOR_KC, "int").reshape(B, T, D)
    w = synth.weights(B * S * H, seed, synth.TENSOR_W, "pow2").reshape(B, S, H)
    return {"q": q, "kc": kc, "w": w}


def _gauss_inputs(B, S, T, seed, H=64, D=128):
    sig = 1 / np.sqrt(D)
    q = synth.matrix(B * S * H, D, seed, synth.TENSOR_Q, "gauss", sig).reshape(B, S, H, D)
    kc = synth.matrix(B * T, D, seed, synth.TENSOR_KC, "gauss", sig).reshape(B, T, D)
    w = synth.weights(B * S * H, seed, synth.TENSOR_W, "uniform", 1 / np.sqrt(H)).reshape(B, S, H)
    return {"q": q, "kc": kc, "w": w}


# ---------------------------------------------------------------- exact cases
@pytest.mark.parametrize("B,S,T,m,k,kw", [
    (1, 256, 64, 4, 16, {}),                       # one diagonal tile, k < n
    (1, 1024, 256, 4, 64, {}),                     # several key tiles
    (1, 1027, 256, 4, 64, {}),                     # ragged query tail (S % 4 != 0)
    (2, 512, 128, 4, 40, {}),                      # two sequences
    (1, 600, 100, 4, 64, {}),                      # T < S/m: rows past 4T see all T keys
    (1, 300, 200, 4, 64, {}),                      # T > S/m: trailing keys never visible
    (1, 512, 512, 1, 100, {}),                     # m = 1
    (1, 513, 171, 3, 37, {}),                      # m = 3, odd sizes
    (1, 1024, 256, 4, 300, {}),                    # k > visible keys for most rows
    (1, 1024, 256, 4, 1, {}),                      # k = 1
    (1, 2048, 512, 4, 2048, {"key_tile": 128}),    # k = 2048 (max)
    (1, 1024, 256, 4, 64, {"key_tile": 64}),       # 64-key partitions
    (1, 2048, 512, 4, 64, {"key_tile": 1024}),     # 1024-key partitions
    (1, 1024, 256, 4, 64, {"query_chunk": 256}),   # chunk driver, 4 launches
    (1, 1536, 384, 4, 96, {"key_tile": 384}),     # partition of 3 tiles (128-key hand-offs)
    (1, 1020, 255, 4, 64, {"query_chunk": 100}),   # ragged chunks
])
def test_integer_inputs_bit_exact(B, S, T, m, k, kw):
    inp = _int_inputs(B, S, T, seed=7 + S + T + k)
    gi, gs = _run(inp, m, k, **kw)
    rows = np.arange(B * S)
    oi, osc, _ = oracle.topk(inp["q"], inp["kc"], inp["w"], m, k)
    parity.check_structure(gi, gs, rows, S, T, m)
    parity.compare_exact(gi, gs, oi, osc, rows)


def test_all_zero_scores_return_first_indices():
    inp = _int_inputs(1, 512, 128, seed=3)
    inp["w"][:] = 0.0
    gi, gs = _run(inp, 4, 32)
    for t in range(512):
        n = min(128, (t + 1) // 4)
        want = np.full(32, -1)
        want[: min(32, n)] = np.arange(min(32, n))
        assert np.array_equal(gi[t], want), t
        assert np.all(gs[t, : min(32, n)] == 0.0)


@pytest.mark.parametrize("key_tile", [64, 128, 256, 1024])
def test_topk_is_a_prefix_of_larger_k(key_tile):
    """Scores do not depend on k, so an exact top-k is a prefix of every
    larger top-k of the same inputs -- bit for bit, at any size, on Gaussian
    inputs too."""
    wl = synth.WORKLOADS["sweep"]
    inp = synth.make_inputs(wl, S=8192)
    kmax = 2048 if key_tile <= 256 else 1024  # k=2048 with 1024-key partitions exceeds shared memory
    ref_i, ref_s = _run(inp, wl.m, kmax, key_tile=key_tile)
    for k in (1, 16, 64, 128, 512, 1024):
        if k >= kmax:
            continue
        gi, gs = _run(inp, wl.m, k, key_tile=key_tile)
        bad = np.nonzero(np.any(gi != ref_i[:, :k], axis=1) | np.any(gs != ref_s[:, :k], axis=1))[0]
        assert len(bad) == 0, (k, len(bad), int(bad[0]), gi[bad[0], -4:], ref_i[bad[0], k - 4:k + 2],
                               gs[bad[0], -4:], ref_s[bad[0], k - 4:k + 2])


def test_materialize_matches_oracle_exactly():
    inp = _int_inputs(1, 1024, 256, seed=5)
    gi, gs = _mat(inp, 4, 64)
    oi, osc, _ = oracle.topk(inp["q"], inp["kc"], inp["w"], 4, 64)
    parity.compare_exact(gi, gs, oi, osc, np.arange(1024))


# ---------------------------------------------------------------- workloads
def test_tiny_gaussian_workload():
    wl = synth.WORKLOADS["tiny"]
    inp = synth.make_inputs(wl)
    gi, gs = _run(inp, wl.m, wl.k)
    rows = np.arange(wl.S)
    oi, _, osc64 = oracle.topk(inp["q"], inp["kc"], inp["w"], wl.m, wl.k)
    parity.check_structure(gi, gs, rows, wl.S, wl.T, wl.m)
    fn = lambda r: oracle.scores(inp["q"], inp["kc"], inp["w"], wl.m, r)  # noqa: E731
    st = parity.compare_tolerant(gi, gs, oi, osc64, rows, fn)
    mi, ms = _mat(inp, wl.m, wl.k)
    st2 = parity.compare_tolerant(gi, gs, mi, ms.astype(np.float64), rows, fn)
    parity.report("workload_recall", "tiny", {"stream_vs_oracle": st, "stream_vs_materialize": st2})
    parity.assert_recall((st, "stream vs oracle"), (st2, "stream vs materialize"))


def test_integer_workload_bit_exact():
    """S=8192, k=512, integer inputs: streaming == oracle == materialize, bit for bit."""
    wl = synth.WORKLOADS["integer"]
    inp = synth.make_inputs(wl)
    gi, gs = _run(inp, wl.m, wl.k)
    rows = np.arange(wl.S)
    oi, osc, _ = parity.oracle_rows("integer", rows, wl.k)
    parity.check_structure(gi, gs, rows, wl.S, wl.T, wl.m)
    parity.compare_exact(gi, gs, oi, osc, rows)
    mi, ms = _mat(inp, wl.m, wl.k)
    parity.compare_exact(mi, ms, oi, osc, rows)


@pytest.fixture(scope="module")
def sweep_oracle():
    wl = synth.WORKLOADS["sweep"]
    rows = np.arange(wl.S)
    return parity.oracle_rows("sweep", rows, 1024)  # prefixes serve every k <= 1024


@pytest.mark.parametrize("axis,value", [(a, v) for a in ("query_chunk", "key_tile", "k")
                                        for v in synth.WORKLOADS["sweep"].sweep[a]])
def test_design_space_sweep(axis, value, sweep_oracle):
    """One cell of the three 5-point sweeps (query chunk, key tile, k): all
    16,384 rows against the oracle and against the materialize path, on plain
    set-overlap recall (mean >= 0.9999, min >= 0.998 in every cell)."""
    wl = synth.WORKLOADS["sweep"]
    inp = synth.make_inputs(wl)
    k = value if axis == "k" else wl.k
    kw = {axis: value} if axis != "k" else {}
    gi, gs = _run(inp, wl.m, k, **kw)
    rows = np.arange(wl.S)
    oi, _, osc64 = (a[:, :k] for a in sweep_oracle)
    parity.check_structure(gi, gs, rows, wl.S, wl.T, wl.m)
    fn = lambda r: oracle.scores(inp["q"], inp["kc"], inp["w"], wl.m, r)  # noqa: E731
    st = parity.compare_tolerant(gi, gs, oi, osc64, rows, fn)
    # the materialize path sums in another fp32 order: every index the two
    # disagree on must lie inside the tie window
    mi, ms = _mat(inp, wl.m, k)
    st2 = parity.compare_tolerant(gi, gs, mi, ms.astype(np.float64), rows, fn)
    st3 = parity.compare_tolerant(mi, ms, oi, osc64, rows, fn)
    parity.report("sweep_recall", f"{axis}={value}",
                  {"stream_vs_oracle": st, "stream_vs_materialize": st2, "materialize_vs_oracle": st3})
    parity.assert_recall((st, f"{axis}={value} stream vs oracle"),
                         (st2, f"{axis}={value} stream vs materialize"),
                         (st3, f"{axis}={value} materialize vs oracle"))


def _full_scores(inp, m, r, T, fmt):
    """Oracle scores of every key of flat row r (NaN for invisible keys)."""
    if fmt == "bf16":
        return oracle.scores(inp["q"], inp["kc"], inp["w"], m, r)
    ii, _, s64 = oracle.topk(inp["q"], inp["kc"], inp["w"], m, T, rows=[r],
                             q_scale=inp["q_scale"], kc_scale=inp["kc_scale"])
    full = np.full(T, np.nan)
    v = ii[0] >= 0
    full[ii[0][v]] = s64[0][v]
    return full


def _sampled(wl, gi, gs, inp, fmt="bf16"):
    rows = synth.sample_rows(254, wl.m - 1, wl.S, seed=wl.seed)
    first_full = wl.m * wl.k - 1  # first row with n >= k
    rows = np.unique(np.concatenate([rows, [first_full, wl.S - 1]]))
    oi, _, osc64 = parity.oracle_rows(wl.name, rows, wl.k, fmt=fmt)
    parity.check_structure(gi[rows], gs[rows], rows, wl.S, wl.T, wl.m)

    def fn(r):
        return _full_scores(inp, wl.m, r, wl.T, fmt)

    return parity.compare_tolerant(gi[rows], gs[rows], oi, osc64, rows, fn)


def test_v4flash_sampled_rows():
    """S=65536, k=512 planted-boost inputs; 256 sampled rows against the oracle."""
    wl = synth.WORKLOADS["v4flash"]
    inp = synth.make_inputs(wl)
    gi, gs = _run(inp, wl.m, wl.k)
    st = _sampled(wl, gi, gs, inp)
    parity.report("workload_recall", "v4flash", {"stream_vs_oracle": st})
    parity.assert_recall((st, "v4flash stream vs oracle"))


def test_materialize_refuses_v4flash_shape():
    """The [1, 65536, 64, 16384] fp32 logits (256 GiB) exceed B200 memory: the
    materialize path refuses with SI_ERR_OUT_OF_MEMORY instead of faulting."""
    wl = synth.WORKLOADS["v4flash"]
    q = torch.zeros((1, wl.S, wl.H, wl.D), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((1, wl.T, wl.D), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((1, wl.S, wl.H), dtype=torch.float32, device="cuda")
    with pytest.raises(si.SIError) as e:
        si.indexer_materialize(q, kc, w, wl.m, wl.k)
    assert e.value.status == si.SI_ERR_OUT_OF_MEMORY


def test_bounded_wait_timeout_is_reported_and_context_survives():
    inp = _int_inputs(1, 1024, 256, seed=11)
    q, kc, w = _dev(inp)
    out = torch.empty((1, 1024, 64), dtype=torch.int32, device="cuda")
    assert si.test_stream_timeout(q, kc, w, 4, 64, out, wait_limit_ns=50_000_000) == si.SI_OK
    assert si.device_status() == si.SI_ERR_TIMEOUT
    assert si.device_status() == si.SI_OK  # record cleared
    gi, gs = _run(inp, 4, 64)  # the context still works
    oi, osc, _ = oracle.topk(inp["q"], inp["kc"], inp["w"], 4, 64)
    parity.compare_exact(gi, gs, oi, osc, np.arange(1024))


def test_unsupported_shapes_are_refused():
    q = torch.zeros((1, 64, 32, 128), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((1, 16, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((1, 64, 32), dtype=torch.float32, device="cuda")
    with pytest.raises(si.SIError) as e:
        si.indexer_topk(q, kc, w, 4, 8)
    assert e.value.status == si.SI_ERR_UNSUPPORTED


# ------------------------------------------------------------ output ordering
def test_unsorted_option_gives_the_same_rows():
    """unsorted=True: each row holds the same entries, valid ones first; the
    row sort entry point then restores the default order exactly."""
    inp = _int_inputs(1, 2048, 512, seed=31)
    q, kc, w = _dev(inp)
    k = 200
    si_idx, si_sc = si.indexer_topk(q, kc, w, 4, k)
    ui, us = si.indexer_topk(q, kc, w, 4, k, unsorted=True)
    assert si.device_status() == si.SI_OK
    a_i, a_s = si_idx.cpu().numpy().reshape(-1, k), si_sc.cpu().numpy().reshape(-1, k)
    b_i, b_s = ui.cpu().numpy().reshape(-1, k), us.cpu().numpy().reshape(-1, k)
    for r in range(a_i.shape[0]):
        nv = int((a_i[r] >= 0).sum())
        assert np.all(b_i[r, :nv] >= 0) and np.all(b_i[r, nv:] == -1)
        assert sorted(zip(a_i[r, :nv], a_s[r, :nv])) == sorted(zip(b_i[r, :nv], b_s[r, :nv]))
    si.sort_topk_rows(ui, us)
    assert si.device_status() == si.SI_OK
    assert np.array_equal(ui.cpu().numpy().reshape(-1, k), a_i)
    assert np.array_equal(us.cpu().numpy().reshape(-1, k), a_s)


def test_without_scores_rows_come_sorted():
    """out_score omitted: the kernel sorts each row itself before storing."""
    inp = _int_inputs(1, 2048, 512, seed=32)
    q, kc, w = _dev(inp)
    for k in (64, 300, 512):
        gi, gs = si.indexer_topk(q, kc, w, 4, k, with_score=False)
        assert gs is None and si.device_status() == si.SI_OK
        oi, _, _ = oracle.topk(inp["q"], inp["kc"], inp["w"], 4, k)
        assert np.array_equal(gi.cpu().numpy().reshape(-1, k), oi)


@pytest.mark.parametrize("k", [1, 7, 64, 100, 257, 301, 512, 1000, 2048])
def test_row_sort_matches_lexicographic_order(k):
    """si_sort_topk_rows on arbitrary rows: score descending, index ascending,
    (-1, -inf) padding last; -0.0 ranks with +0.0."""
    rng = np.random.default_rng(k)
    rows = 300
    idx = rng.permutation(rows * k).astype(np.int32).reshape(rows, k)
    sc = rng.choice(np.float32([-2.5, -0.0, 0.0, 1.0, 1.0, 3.25, 7.0]), size=(rows, k))
    sc += rng.integers(0, 3, size=(rows, k)).astype(np.float32) * (rng.random((rows, k)) < 0.5)
    pad = rng.random((rows, k)) < 0.1
    idx[pad] = -1
    sc[pad] = -np.inf
    ti, ts = torch.from_numpy(idx).cuda(), torch.from_numpy(sc).cuda()
    si.sort_topk_rows(ti, ts)
    assert si.device_status() == si.SI_OK
    gi, gs = ti.cpu().numpy(), ts.cpu().numpy()
    for r in range(rows):
        # padding sorts last: give it the lowest rank explicitly
        s = np.where(idx[r] < 0, -np.inf, sc[r]).astype(np.float64) + 0.0  # -0.0 -> 0.0
        key_idx = np.where(idx[r] < 0, np.iinfo(np.int64).max, idx[r].astype(np.int64))
        order = np.lexsort((key_idx, -s))
        assert np.array_equal(gi[r], idx[r][order]), r
        assert np.array_equal(np.abs(gs[r]), np.abs(sc[r][order])), r


@pytest.mark.parametrize("k", [257, 384, 512])
@pytest.mark.parametrize("kind", ["gauss", "narrow", "early_rows"])
def test_row_sort_distinct_and_clustered_scores(k, kind):
    """si_sort_topk_rows on rows whose scores are mostly distinct (the shape
    the streaming kernel hands over): Gaussian, a narrow cluster with a few
    outliers and exact ties, and early-row shapes with a long padding tail.
    Score descending, index ascending, (-1, -inf) padding last."""
    rng = np.random.default_rng(1000 + k)
    rows = 256
    idx = rng.permutation(rows * k).astype(np.int32).reshape(rows, k)
    if kind == "gauss":
        sc = rng.standard_normal((rows, k)).astype(np.float32)
    else:
        sc = (5.0 + 1e-3 * rng.standard_normal((rows, k))).astype(np.float32)
        sc[:, :3] = np.float32([40.0, -7.0, 5.0])
    tie = rng.random((rows, k)) < 0.05
    sc[tie] = sc[:, :1].repeat(k, axis=1)[tie]  # exact ties with the row's first score
    if kind == "early_rows":
        n_real = rng.integers(0, k + 1, size=rows)
        pad = np.arange(k)[None, :] >= n_real[:, None]
    else:
        pad = rng.random((rows, k)) < 0.1
    idx[pad] = -1
    sc[pad] = -np.inf
    ti, ts = torch.from_numpy(idx).cuda(), torch.from_numpy(sc).cuda()
    si.sort_topk_rows(ti, ts)
    assert si.device_status() == si.SI_OK
    gi, gs = ti.cpu().numpy(), ts.cpu().numpy()
    for r in range(rows):
        s = np.where(idx[r] < 0, -np.inf, sc[r]).astype(np.float64) + 0.0
        key_idx = np.where(idx[r] < 0, np.iinfo(np.int64).max, idx[r].astype(np.int64))
        order = np.lexsort((key_idx, -s))
        assert np.array_equal(gi[r], idx[r][order]), r
        assert np.array_equal(gs[r], sc[r][order]), r


def test_default_key_tile_falls_back_for_large_k():
    """k=2048 with the default partition: the library picks a partition whose
    pool fits (an explicit 512 is refused) and the result is exact."""
    inp = _int_inputs(1, 2048, 512, seed=33)
    q, kc, w = _dev(inp)
    with pytest.raises(si.SIError) as e:
        si.indexer_topk(q, kc, w, 4, 2048, key_tile=512)
    assert e.value.status == si.SI_ERR_UNSUPPORTED
    gi, gs = _run(inp, 4, 2048)
    oi, osc, _ = oracle.topk(inp["q"], inp["kc"], inp["w"], 4, 2048)
    parity.compare_exact(gi, gs, oi, osc, np.arange(2048))


@pytest.mark.parametrize("B,S,T,bounds", [
    (1, 2048, 512, [0, 512, 1100, 2048]),        # chunks, one not a multiple of 4
    (2, 1030, 256, [0, 3, 517, 1030]),           # two sequences, tiny first chunk
])
def test_row_ranges_equal_the_whole_sequence(B, S, T, bounds):
    """Rows fed in chunks through si_indexer_topk_rows give exactly the rows of
    the whole-sequence call (integer inputs: bit for bit, also vs the oracle)."""
    inp = _int_inputs(B, S, T, seed=41 + S)
    q, kc, w = _dev(inp)
    k = 96
    gi, gs = si.indexer_topk(q, kc, w, 4, k)
    parts_i, parts_s = [], []
    for r0, r1 in zip(bounds[:-1], bounds[1:]):
        ci, cs = si.indexer_topk_rows(q[:, r0:r1].contiguous(), kc, w[:, r0:r1].contiguous(), 4, k, r0)
        parts_i.append(ci)
        parts_s.append(cs)
    assert si.device_status() == si.SI_OK
    ri, rs = torch.cat(parts_i, dim=1), torch.cat(parts_s, dim=1)
    assert torch.equal(ri, gi) and torch.equal(rs, gs)
    oi, osc, _ = oracle.topk(inp["q"], inp["kc"], inp["w"], 4, k)
    parity.compare_exact(ri.cpu().numpy().reshape(-1, k), rs.cpu().numpy().reshape(-1, k), oi, osc,
                         np.arange(B * S))


@pytest.mark.parametrize("parts", [2, 3, 8])
def test_row_shards_put_together_equal_the_whole_sequence(parts):
    """The row partition a multi-GPU run uses (equal visible pairs per part),
    run part by part on one GPU through si_indexer_topk_rows, gives the
    whole-sequence rows bit for bit (integer inputs)."""
    B, S, T, k = 1, 4096, 1024, 128
    inp = _int_inputs(B, S, T, seed=77 + parts)
    q, kc, w = _dev(inp)
    gi, gs = si.indexer_topk(q, kc, w, 4, k)
    bounds = si.row_shards(S, T, 4, parts)
    pi, ps = [], []
    for r0, r1 in zip(bounds[:-1], bounds[1:]):
        ci, cs = si.indexer_topk_rows(q[:, r0:r1].contiguous(), kc, w[:, r0:r1].contiguous(), 4, k, r0)
        pi.append(ci)
        ps.append(cs)
    assert si.device_status() == si.SI_OK
    assert torch.equal(torch.cat(pi, dim=1), gi) and torch.equal(torch.cat(ps, dim=1), gs)
