"""The seeded input generator (no GPU)."""
import numpy as np
import pytest
import torch

import synth


def test_splitmix64_reference_values():
    # SplitMix64 seeded with 0: the first outputs of the published generator
    L = synth.lib()
    assert L.synth_draw(0, 0) == 0xE220A8397B1DCDAF
    assert L.synth_draw(0, 1) == 0x6E789E6AA1B965F4
    assert L.synth_draw(0, 2) == 0x06C45D188009454F


def test_deterministic_and_counter_based():
    a = synth.matrix(300, 128, seed=5, tensor_id=1)
    b = synth.matrix(300, 128, seed=5, tensor_id=1)
    c = synth.matrix(300, 128, seed=6, tensor_id=1)
    d = synth.matrix(300, 128, seed=5, tensor_id=2)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c) and not np.array_equal(a, d)
    big = synth.matrix(20000, 128, seed=5, tensor_id=1)  # threaded path
    assert np.array_equal(big[:300], a)


def test_gaussian_moments():
    x = synth.bf16_bits_to_f32(synth.matrix(4096, 128, seed=1, tensor_id=1, sigma=1 / np.sqrt(128)))
    assert abs(x.mean()) < 2e-3
    assert abs(x.std() * np.sqrt(128) - 1.0) < 5e-3
    z = x.ravel() * np.sqrt(128)
    assert abs((z ** 4).mean() - 3.0) < 0.05  # Gaussian kurtosis


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(200000) * 10.0 ** rng.integers(-8, 8, 200000)).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(synth.f32_to_bf16_bits(x), want)
    L = synth.lib()
    got = np.array([L.synth_f32_to_bf16(float(v)) for v in x[:5000]], dtype=np.uint16)
    assert np.array_equal(got, want[:5000])


def test_e4m3_rounding_matches_torch():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(20000) * 2.0 ** rng.integers(-12, 9, 20000)).astype(np.float32)
    x = np.clip(x, -448.0, 448.0)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    L = synth.lib()
    got = np.array([L.synth_f32_to_e4m3(float(v)) for v in x], dtype=np.uint8)
    assert np.array_equal(got, want)
    assert L.synth_f32_to_e4m3(1000.0) == 0x7E and L.synth_f32_to_e4m3(-1e9) == 0xFE


def test_e4m3_rows_dequantise_close():
    q8, s = synth.matrix(512, 128, seed=3, tensor_id=1, sigma=1 / np.sqrt(128), fmt="e4m3")
    xf = synth.bf16_bits_to_f32(synth.matrix(512, 128, seed=3, tensor_id=1, sigma=1 / np.sqrt(128)))
    deq = torch.from_numpy(q8).view(torch.float8_e4m3fn).float().numpy() * s[:, None]
    assert np.abs(deq).max(axis=1).max() <= np.abs(xf).max() * 1.01
    rel = np.abs(deq - xf) / (np.abs(xf).max(axis=1, keepdims=True))
    assert rel.max() < 2 ** -4 + 1e-2  # 3 mantissa bits
    assert np.all(np.abs(deq).max(axis=1) == np.float32(448.0) * s)  # amax maps to 448


def test_integer_and_pow2():
    x = synth.bf16_bits_to_f32(synth.matrix(1000, 128, seed=1, tensor_id=1, kind="int"))
    assert set(np.unique(x).tolist()) == set(range(-3, 4))
    w = synth.weights(100000, seed=1, tensor_id=3, kind="pow2")
    assert set(np.unique(w).tolist()) == {2.0 ** -j for j in range(7)}
    u = synth.weights(100000, seed=1, tensor_id=3, kind="uniform", scale=0.125)
    assert u.min() >= 0.0 and u.max() < 0.125 and abs(u.mean() - 0.0625) < 1e-3


def test_planted_keys():
    T, D = 4096, 128
    (kc, mask) = synth.keys_planted(2, T, D, seed=3, tensor_id=2, sigma=1 / np.sqrt(D), frac=0.05,
                                    boost=2.0, with_mask=True)
    mask = mask.reshape(2, T)
    assert np.all(mask.sum(axis=1) == round(0.05 * T))
    x = synth.bf16_bits_to_f32(kc).reshape(2, T, D)
    nb = np.linalg.norm(x[mask == 1], axis=1)
    nu = np.linalg.norm(x[mask == 0], axis=1)
    assert abs(nu.mean() - 1.0) < 0.02 and nb.mean() > 2.0  # |z + 2u| ~ sqrt(1 + 4)
    plain = synth.bf16_bits_to_f32(synth.matrix(2 * T, D, seed=3, tensor_id=2, sigma=1 / np.sqrt(D)))
    assert np.array_equal(x.reshape(-1, D)[mask.ravel() == 0], plain[mask.ravel() == 0])


def test_sample_rows():
    r = synth.sample_rows(256, 3, 65536, seed=3)
    assert len(np.unique(r)) == 256 and r.min() >= 3 and r.max() < 65536
    assert np.all(np.diff(r) > 0)
    assert np.array_equal(r, synth.sample_rows(256, 3, 65536, seed=3))


def test_visible_pairs_closed_form():
    for S, T, m in [(1024, 256, 4), (8192, 2048, 4), (30, 8, 4), (17, 16, 1), (100, 7, 3)]:
        brute = sum(min(T, (t + 1) // m) for t in range(S))
        assert synth.visible_pairs(S, T, m) == brute
    wl = synth.WORKLOADS["v4flash"]
    assert wl.visible_pairs() == 536854528
    assert synth.WORKLOADS["million"].visible_pairs() == 137438691328


@pytest.mark.parametrize("name,fmt", [("tiny", "bf16"), ("tiny", "e4m3"), ("integer", "bf16"),
                                      ("integer", "e4m3")])
def test_rows_generated_alone_equal_the_full_tensor(name, fmt):
    """q_rows / make_inputs_rows give exactly the rows of make_inputs."""
    wl = synth.WORKLOADS[name]
    full = synth.make_inputs(wl, fmt=fmt)
    rows = np.array([0, 5, 777, wl.S - 1])
    part = synth.make_inputs_rows(wl, rows, fmt=fmt)
    for r in rows:
        assert np.array_equal(full["q"][0, r], part["q"][0, r])
        if fmt != "bf16":
            assert np.array_equal(full["q_scale"][0, r], part["q_scale"][0, r])
    assert np.array_equal(full["kc"], part["kc"]) and np.array_equal(full["w"], part["w"])
    blk = synth.q_rows(wl, 0, 100, 37, fmt)
    if fmt == "bf16":
        assert np.array_equal(blk, full["q"][0, 100:137])
    else:
        assert np.array_equal(blk[0], full["q"][0, 100:137])
        assert np.array_equal(blk[1], full["q_scale"][0, 100:137])
