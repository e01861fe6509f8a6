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


def test_mxfp4_widening_all_codes(oracle_lib):
    """E2M1 codes and E8M0 scales against ml_dtypes' OCP MX conversions."""
    import ml_dtypes
    codes = np.arange(16, dtype=np.uint8)
    want = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    got = np.array([oracle_lib.oracle_e2m1_value(int(c)) for c in codes])
    assert np.array_equal(got, want) and np.array_equal(np.signbit(got), np.signbit(want))
    sc = np.arange(256, dtype=np.uint8)
    want = sc.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    got = np.array([oracle_lib.oracle_e8m0_value(int(c)) for c in sc])
    assert np.array_equal(np.isnan(got), np.isnan(want))
    fin = ~np.isnan(want)
    assert np.array_equal(got[fin], want[fin])
    assert oracle_lib.oracle_e2m1_value(7) == 6.0 and oracle_lib.oracle_e8m0_value(127) == 1.0


def test_mxfp4_quantiser_round_trip(oracle_lib):
    """The input generator's MXFP4 quantiser: values already on a block's
    grid come back unchanged through the oracle's decode, and every block
    scale puts the block's largest magnitude in [4, 8) before saturation."""
    rng = np.random.default_rng(5)
    import ml_dtypes
    codes = rng.integers(0, 16, size=(64, 128)).astype(np.uint8)
    codes[:, ::32] = 7  # a +6 in every block fixes its scale
    e = rng.integers(-20, 20, size=(64, 4))
    vals = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64) * np.ldexp(1.0, e).repeat(32, axis=-1)
    packed, scales = synth.quantize_mxfp4(vals.astype(np.float32))
    assert np.array_equal(scales.astype(np.int64) - 127, e)
    assert np.array_equal(oracle.mxfp4_decode(packed, scales, lib=oracle_lib), vals)
    x = rng.standard_normal((32, 128)).astype(np.float32)
    _, sc = synth.quantize_mxfp4(x)
    amax = np.abs(x.reshape(32, 4, 32)).max(-1) / np.ldexp(1.0, sc.astype(np.int64) - 127)
    assert np.all((amax >= 4) & (amax < 8))


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
