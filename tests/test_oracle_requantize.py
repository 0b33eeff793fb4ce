"""Pins of the oracle's tier demotion (re-quantising a page from the values read back)."""
import numpy as np
import pytest

from oracle import cache as ocache
from oracle.layout import T
from oracle.quant import TIER_F8, TIER_F16, TIER_I1, TIER_I2, TIER_I4, TIER_I8, quantise_token
from sparse_mixed_precision_kvq_b200 import workloads as W


def _head(tiers, L=100, seed=0, dtype="bf16"):
    rng = np.random.default_rng(seed)
    x = rng.normal(0, 1, (2, L, 64)).astype(np.float32)
    x[:, :, 5] *= 8.0
    bits = W.f32_to_bf16_bits(x) if dtype == "bf16" else x.astype(np.float16).view(np.uint16)
    return ocache.build(bits[0], bits[1], dtype, np.asarray(tiers)), bits


@pytest.mark.parametrize("tier", [TIER_F8, TIER_I8, TIER_I4, TIER_I2, TIER_I1])
def test_demoting_a_16bit_page_equals_storing_it_at_the_tier(tier):
    """A 16-bit page reads back its original values, so demoting it must give the bytes
    of the same page stored at the lower tier from the start."""
    P = 7
    sh16, bits = _head([TIER_F16] * P)
    direct, _ = _head([TIER_F16] * 3 + [tier] + [TIER_F16] * 3)
    ocache.requantize(sh16, 3, tier)
    for kind in "kv":
        assert np.array_equal(ocache.page_bytes(sh16, 3, kind), ocache.page_bytes(direct, 3, kind))
    assert np.array_equal(sh16.khat[3 * T:4 * T], direct.khat[3 * T:4 * T])
    assert np.array_equal(sh16.summary, direct.summary)  # the summary does not move


@pytest.mark.parametrize("src,dst", [(TIER_I8, TIER_I4), (TIER_I8, TIER_I1), (TIER_I4, TIER_I2), (TIER_I2, TIER_I1),
                                     (TIER_F8, TIER_I4), (TIER_F8, TIER_I1)])
def test_demoting_a_quantised_page_requantises_its_read_back_values(src, dst):
    P = 7
    sh, _ = _head([src] * P, L=16 * P - 3, seed=2)
    old = sh.khat.copy(), sh.vhat.copy()
    ocache.requantize(sh, P - 1, dst)           # a partial last page: 13 tokens
    for t in range(16 * (P - 1), sh.L):
        q = quantise_token(old[0][t].copy(), dst)
        assert np.array_equal(sh.kcodes[t], q["codes"]) and np.array_equal(sh.kmeta[t], q["meta"])
        if dst not in (TIER_I1, TIER_F8):  # the round-trip bound of the second quantisation
            sc = np.array([float(np.float16(np.uint16(m & 0xFFFF).view(np.float16))) for m in q["meta"]])
            err = np.abs(sh.khat[t] - old[0][t]).reshape(-1, 32).max(1)
            assert np.all(err <= sc / 2 * (1 + 1e-6) + 1e-3 * sc)
    assert int(sh.tiers[P - 1]) == dst
    assert np.array_equal(sh.khat[:16 * (P - 1)], old[0][:16 * (P - 1)])  # other pages untouched


def test_demotion_never_grows_the_page():
    sh, _ = _head([TIER_F16] * 5)
    sizes = []
    for tier in (TIER_I8, TIER_I4, TIER_I2, TIER_I1):  # (fp8's 2-byte scales make it smaller than int8)
        ocache.requantize(sh, 2, tier)
        sizes.append(ocache.page_bytes(sh, 2, "k").size)
    assert sizes == sorted(sizes, reverse=True)
