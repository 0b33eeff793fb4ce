"""The re-quantiser's fp32 route decides every integer code exactly as the fp64 quantiser.

The demotion kernel computes q = (x - zero) * (1 / scale) in fp32 (single IEEE operations;
its unit is built without fused multiply-add), takes rint(q), and falls back to the exact
fp64 quotient only when q lies within 1e-4 of a rounding tie or is not finite.  This test
replays that decision in numpy float32 (the same single roundings) on random groups,
requantised values, and groups built to sit just off ties, and checks each code against
the oracle's quantiser (fp64 quotient, round half to even, clamp)."""
import numpy as np
import pytest

from oracle.quant import GROUP, quantise_int


def _fast_codes(x32: np.ndarray, bits: int):
    """Codes of groups x32 [n, 32] (float32) by the kernel's route."""
    qmax = (1 << bits) - 1
    _, scale, zero, *_ = quantise_int(x32.astype(np.float64), bits)   # the fp64 metadata (shared step)
    zf = zero.astype(np.float32)[:, None]
    sf = scale.astype(np.float32)[:, None]
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        inv = np.float32(1.0) / sf
        q = (x32 - zf) * inv
        r = np.rint(q)
        near = ~(np.abs(q - r) < np.float32(0.4999))
        exact = np.rint((x32.astype(np.float64) - zf.astype(np.float64)) / sf.astype(np.float64))
    c = np.where(near, exact, r.astype(np.float64))
    c = np.clip(np.nan_to_num(c, nan=0.0), 0, qmax)
    c = np.where(sf == 0, 0, c)
    return c.astype(np.int64), near


@pytest.mark.parametrize("bits", [8, 4, 2])
def test_random_and_requantised_groups(bits):
    rng = np.random.default_rng(bits)
    n = 20000
    x = rng.standard_normal((n, GROUP)) * rng.uniform(1e-3, 1e3, (n, 1)) + rng.normal(0, 5, (n, 1))
    x32 = x.astype(np.float32)
    want = quantise_int(x32.astype(np.float64), bits)[0]
    got, _ = _fast_codes(x32, bits)
    assert np.array_equal(got, want)
    # values read back from an 8-bit tier (fp32(c*scale + zero)) quantised again
    c8, s8, z8, *_ = quantise_int(x32.astype(np.float64), 8)
    back = (c8 * s8[:, None] + z8[:, None]).astype(np.float32)
    want2 = quantise_int(back.astype(np.float64), bits)[0]
    got2, _ = _fast_codes(back, bits)
    assert np.array_equal(got2, want2)


@pytest.mark.parametrize("bits", [8, 4, 2])
def test_groups_built_around_ties(bits):
    """x = zero + (k + 1/2 + e) * scale with |e| from 1e-9 to 1e-2: the route takes the exact
    path near ties and agrees with the fp64 quantiser everywhere."""
    rng = np.random.default_rng(100 + bits)
    qmax = (1 << bits) - 1
    n = 20000
    lo = rng.normal(0, 3, n).astype(np.float16).astype(np.float64)       # exact fp16 zero
    sc = rng.uniform(0.01, 0.5, n).astype(np.float16).astype(np.float64)  # exact fp16 scale
    k = rng.integers(0, qmax, (n, GROUP))
    e = rng.choice([-1, 1], (n, GROUP)) * 10.0 ** rng.uniform(-9, -2, (n, GROUP))
    x = lo[:, None] + (k + 0.5 + e) * sc[:, None]
    x[:, 0] = lo                          # pin the group's min and max so that the
    x[:, 1] = lo + qmax * sc              # metadata comes out as (lo, sc) when exact
    x32 = x.astype(np.float32)
    want = quantise_int(x32.astype(np.float64), bits)[0]
    got, near = _fast_codes(x32, bits)
    assert np.array_equal(got, want)
    assert near.mean() > 0.01             # the exact route was exercised
