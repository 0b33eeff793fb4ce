"""The seeded input generators: determinism, shapes and the recipe of each workload."""
import numpy as np

from sparse_mixed_precision_kvq_b200 import workloads as W


def test_deterministic_and_sliceable():
    w = W.small("c1")
    a, b = w.keys_bits(1, 3), W.small("c1").keys_bits(1, 3)
    assert np.array_equal(a, b) and a.shape == (2048, 128) and a.dtype == np.uint16
    assert not np.array_equal(w.keys_bits(0, 3), a)


def test_full_shapes_and_budgets():
    c1, c2, c3, c4 = (W.make(n) for n in ("c1", "c2", "c3", "c4"))
    assert (c1.B, c1.Hq, c1.Hkv, c1.D, c1.max_pages) == (8, 32, 8, 128, 2049)
    assert c1.kmax() == 103 + 5 and c2.kmax() == 205 + 5 and c3.kmax() == 410 + 17
    assert c3.max_pages == 8193 and c3.plant_count == 410
    assert c4.B == 64 and c4.G == 8 and c4.lens.min() >= 2048 and c4.lens.max() < 65536


def test_tier_ratios_and_new_page():
    w = W.make("c2", B=1)
    t = w.tiers(0)
    assert t.size == 2049 and t[2048] == W.TIER_F16
    counts = np.bincount(t[:2048], minlength=5)
    assert list(counts[:4]) == [204, 410, 614, 820]   # floor of the cumulative fractions


def test_c3_hot_set_is_planted_plus_forced():
    w = W.small("c3")
    t = w.tiers(0)
    hot = set(np.nonzero(t == W.TIER_F16)[0])
    P1 = w.pages_after(0)
    assert hot == set(w.planted_pages(0)) | {0} | set(range(P1 - 16, P1))
    assert np.all(t[list(set(range(P1)) - hot)] == W.TIER_I4)
    tt, st, counts = w.slot_map()
    assert sorted(st[0, tt[0] == W.TIER_I4]) == list(range(counts[W.TIER_I4]))


def test_outliers_and_bf16_rounding():
    w = W.small("c1")
    x = W.bits_to_f32(w.keys_bits(0, 0), "bf16")
    idx = w.outlier_idx(0)
    assert idx.size == 4
    big = np.abs(x[:, idx]).mean()
    rest = np.abs(np.delete(x, idx, axis=1)).mean()
    assert big > 5 * rest
    assert np.array_equal(W.f32_to_bf16_bits(np.array([1 + 2 ** -8], np.float32)), np.array([0x3F80], np.uint16))
    assert np.array_equal(W.f32_to_bf16_bits(np.array([1 + 3 * 2 ** -8], np.float32)), np.array([0x3F82], np.uint16))
