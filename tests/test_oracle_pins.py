"""The CPU oracle against its pins (no GPU)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL, ids=lambda f: f.__name__)
def test_pin(pin, oracle_lib):
    pin(oracle_lib)


def test_bf16_widening_all_codes(oracle_lib):
    codes = np.arange(65536, dtype=np.uint16)
    want = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([oracle_lib.oracle_bf16_value(int(c)) for c in codes])
    fin = np.isfinite(want)
    assert np.array_equal(got[fin], want[fin])
    assert np.array_equal(np.isnan(got), np.isnan(want))


def test_e4m3_widening_all_codes(oracle_lib):
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle_lib.oracle_e4m3_value(int(c)) for c in codes])
    assert np.array_equal(np.isnan(got), np.isnan(want))
    fin = ~np.isnan(want)
    assert np.array_equal(got[fin], want[fin])
    # OCP E4M3 landmarks: max finite 448, min normal 2^-6, min subnormal 2^-9
    assert oracle_lib.oracle_e4m3_value(0x7E) == 448.0
    assert oracle_lib.oracle_e4m3_value(0x08) == 2.0 ** -6
    assert oracle_lib.oracle_e4m3_value(0x01) == 2.0 ** -9
    assert oracle_lib.oracle_e4m3_value(0x38) == 1.0


def test_visible_count_definition(oracle_lib):
    # key s covers tokens [s*m, s*m+m-1]; count keys whose last token <= t
    for m in (1, 2, 3, 4, 7):
        for T in (1, 5, 9):
            for t in range(0, 40):
                n = sum(1 for s in range(T) if s * m + m - 1 <= t)
                assert oracle.visible_count(t, T, m, lib=oracle_lib) == n


def test_integer_workload_is_fp32_exact(oracle_lib):
    """Integer inputs of the integer-exact workload: every oracle score is a
    multiple of 2^-6 below 2^17, so it is exact in fp32."""
    wl = synth.WORKLOADS["integer"]
    inp = synth.make_inputs(wl, S=256)
    idx, sc, sc64 = oracle.topk(inp["q"], inp["kc"], inp["w"], wl.m, 64, lib=oracle_lib)
    v = idx >= 0
    assert np.array_equal(sc[v].astype(np.float64), sc64[v])
    assert np.all(np.abs(sc64[v]) < 2.0 ** 17)
    assert np.all(np.floor(sc64[v] * 64) == sc64[v] * 64)


def test_gaussian_scores_are_finite_and_nonnegative(oracle_lib):
    wl = synth.WORKLOADS["tiny"]
    inp = synth.make_inputs(wl)
    rows = np.array([3, 100, 517, 1023])
    idx, sc, sc64 = oracle.topk(inp["q"], inp["kc"], inp["w"], wl.m, wl.k, rows=rows, lib=oracle_lib)
    v = idx >= 0
    assert np.all(np.isfinite(sc64[v])) and np.all(sc64[v] >= 0.0)  # w >= 0
    for i in range(len(rows)):                                        # sorted descending
        n = int(v[i].sum())
        assert np.all(np.diff(sc64[i, :n]) <= 0.0)
