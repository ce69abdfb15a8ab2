"""Seeded input recipes: determinism, row-range independence, structure, sizes."""

import numpy as np
import pytest
import torch

from hadamard_rotation_bit_b200 import workloads as W


def test_algorithmic_bytes_match_the_configs():
    assert W.WORKLOADS["c1"].algorithmic_bytes == 295_936
    assert W.WORKLOADS["c2"].algorithmic_bytes == 42_205_184
    assert W.WORKLOADS["c3"].algorithmic_bytes == 352_354_304
    assert W.WORKLOADS["c4q"].algorithmic_bytes + W.WORKLOADS["c4k"].algorithmic_bytes == 1_749_024_768
    assert W.WORKLOADS["c5"].algorithmic_bytes == 1_358_954_496


@pytest.mark.parametrize("key", ["c1", "c2", "c4q", "c4k"])
def test_row_ranges_regenerate_identically(key):
    w = W.WORKLOADS[key]
    hi = min(w.rows, 2 * W.CHUNK_ROWS + 7)
    full = W.generate(key, slice(0, hi))
    for lo, up in [(0, 3), (W.CHUNK_ROWS - 2, W.CHUNK_ROWS + 5), (hi - 9, hi)]:
        lo, up = max(0, min(lo, w.rows - 1)), min(up, hi)
        np.testing.assert_array_equal(W.generate(key, slice(lo, up)), full[lo:up])
    ids = np.array([hi - 1, 0, min(W.CHUNK_ROWS, hi - 1), 1])
    np.testing.assert_array_equal(W.generate_rows(key, ids), full[ids])


def test_seeds_differ_and_repeat():
    a = W.generate("c2", slice(0, 8))
    np.testing.assert_array_equal(a, W.generate("c2", slice(0, 8)))
    assert not np.array_equal(a, W.generate("c2", slice(0, 8), seed=W.rank_seed(1)))


def test_bf16_conversion_matches_torch():
    rng = np.random.default_rng(0)
    v = (rng.standard_normal(100_000) * np.exp(rng.uniform(-20, 20, 100_000))).astype(np.float32)
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(W.f32_to_bf16_bits(v), want)
    back = W.bits_to_float64(want, "bf16")
    np.testing.assert_array_equal(back, torch.from_numpy(want.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_c2_outlier_channels():
    x = W.bits_to_float64(W.generate("c2", slice(0, 512)), "bf16")
    rms = np.sqrt((x ** 2).mean(0))
    big = np.sort(np.argsort(rms)[-41:])
    assert rms[big].min() > 20 * np.median(rms)
    assert np.sort(rms)[-42] < 2.0


def test_c3_silu_product_and_outliers():
    x = W.bits_to_float64(W.generate("c3", slice(0, 256)), "bf16")
    rms = np.sqrt((x ** 2).mean(0))
    assert (rms > 10 * np.median(rms)).sum() == 72


def test_c4_rope_and_head_outliers():
    w = W.WORKLOADS["c4k"]
    x = W.bits_to_float64(W.generate("c4k", slice(0, 1024)), "bf16")   # head 0, positions 0..1023
    assert x.shape == (1024, 128)
    # position 0 has no rotation: the two outlier dims stand out directly
    e = np.sqrt((x[:1] ** 2))
    assert (e > 8).sum() <= 2
    # RoPE preserves the pair norms (i, i + 64) position by position
    pn = x[:, :64] ** 2 + x[:, 64:] ** 2
    assert pn.shape == (1024, 64)
    assert w.rows == 16 * 32 * 4096


def test_c5_heavy_tails():
    x = W.bits_to_float64(W.generate("c5", slice(0, 64)), "bf16")
    assert np.abs(x).max() > 30      # Student-t(3) tails
    assert 1.0 < x.std() < 3.0


def test_random_hadamard_workloads_share_the_c2_input():
    for key in ("c2r", "c2rb"):
        w = W.WORKLOADS[key]
        assert w.algorithmic_bytes == W.WORKLOADS["c2"].algorithmic_bytes
        np.testing.assert_array_equal(W.generate(key, slice(1020, 1030)), W.generate("c2", slice(1020, 1030)))
        s = W.generate_signs(key)
        assert s.dtype == np.int8 and s.shape == (w.block,) and set(np.unique(s)) == {-1, 1}
        assert abs(int(s.astype(np.int64).sum())) < 4 * np.sqrt(w.block)       # Rademacher draws
        np.testing.assert_array_equal(s, W.generate_signs(key))
        assert not np.array_equal(s, W.generate_signs(key, seed=W.rank_seed(1)))
    assert W.WORKLOADS["c2r"].signs == "after" and W.WORKLOADS["c2rb"].signs == "before"
    for key, base in (("c3rb", "c3"), ("c5rb", "c5")):
        w, wb = W.WORKLOADS[key], W.WORKLOADS[base]
        assert w.signs == "before" and w.algorithmic_bytes == wb.algorithmic_bytes and w.block == wb.block
        np.testing.assert_array_equal(W.generate(key, slice(0, 3)), W.generate(base, slice(0, 3)))
        assert W.generate_signs(key).shape == (w.block,)
    with pytest.raises(ValueError):
        W.generate_signs("c2")


def test_nvfp4_workloads_share_their_inputs():
    assert W.WORKLOADS["c2n"].algorithmic_bytes == 33_554_432 + 8_388_608 + 4096 * 256
    assert W.WORKLOADS["c5n"].algorithmic_bytes == 1_073_741_824 + 268_435_456 + 65536 * 512
    np.testing.assert_array_equal(W.generate("c2n", slice(5, 9)), W.generate("c2", slice(5, 9)))
    np.testing.assert_array_equal(W.generate("c5n", slice(2047, 2050)), W.generate("c5", slice(2047, 2050)))
