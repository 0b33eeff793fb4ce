"""The attention kernel's exact code -> 16-bit operand conversions, replayed in numpy on
every code (IEEE single roundings, subnormals kept, as the kernels are built):

* integer tiers: the code placed in the mantissa of a 16-bit float with a magic exponent
  (fp16 1024, bf16 128), minus (magic + 2^(b-1)), is the centred code c - 2^(b-1);
* 8-bit codes for bf16 operands: 2^23 + c as fp32, minus 2^23 + 128, is c - 128 (exact in
  bf16, whose 7-bit mantissa cannot hold 128 + c);
* fp8: the e4m3 byte's exponent and mantissa placed in an fp32 pattern and multiplied by
  2^120 give the e4m3 value, subnormals included;
* the selection's score -> order key map is monotone, ranks -0 with +0 and NaN lowest,
  and inverts;
* the score kernels' split of a bf16 query into fp16 high and 2^24-scaled low parts is
  exact for every element of magnitude >= 2^-41."""
import numpy as np

from oracle.quant import e4m3_value


def _f16(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def _bf16(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def test_magic_exponent_centred_codes():
    for b in (8, 4, 2):
        c = np.arange(1 << b)
        centre = 1 << (b - 1)
        f16 = _f16(0x6400 | c) - _f16(0x6400 | centre)          # fp16 subtraction is exact here
        assert np.array_equal(f16, c - centre)
        if b < 8:
            bf = _bf16(0x4300 | c) - _bf16(0x4300 | centre)
            assert np.array_equal(bf, c - centre)
    # why bf16 needs another route at 8 bits: 128 + c is not representable for odd c >= 128
    assert _bf16(0x4300 | 0x81) != 128 + 0x81


def test_fp32_route_for_8bit_codes_in_bf16():
    c = np.arange(256, dtype=np.uint32)
    v = (np.uint32(0x4B000000) | c).view(np.float32) - np.float32(8388736.0)
    assert np.array_equal(v.astype(np.float64), c.astype(np.float64) - 128)
    # every centred value is exact in bf16 (8 significant bits suffice for |c - 128| <= 128)
    as_bf16 = (v.view(np.uint32) >> 16 << 16).view(np.float32)
    assert np.array_equal(as_bf16, v)


def test_e4m3_pattern_times_2_120():
    b = np.arange(256, dtype=np.uint32)
    pattern = (((b & 0x80) << 24) | ((b & 0x7F) << 20)).view(np.float32)
    v = (pattern * np.float32(2.0 ** 120)).astype(np.float64)
    ref = e4m3_value(b)
    fin = np.isfinite(ref)
    assert np.array_equal(v[fin], ref[fin])                       # subnormals: codes 1..7
    assert np.all(np.isfinite(v))                                 # NaN codes come out finite (480)
    # every e4m3 value is exact in bf16 and fp16 operands
    assert np.array_equal(v[fin].astype(np.float16).astype(np.float64), v[fin])
    assert np.array_equal(((v[fin].astype(np.float32).view(np.uint32) >> 16) << 16).view(np.float32), v[fin])


def _order_key(f: np.ndarray) -> np.ndarray:
    """The selection's score -> key map (NaN -> 0, -0 -> +0, then the IEEE order trick)."""
    f = np.where(f == 0, np.float32(0.0), f).astype(np.float32)
    u = f.view(np.uint32)
    k = np.where(u & 0x80000000, ~u, u | 0x80000000).astype(np.uint32)
    return np.where(np.isnan(f), np.uint32(0), k)


def test_selection_order_key_is_monotone_with_nan_lowest():
    fi = np.finfo(np.float32)
    vals = np.array([-np.inf, -fi.max, -1.0, -fi.tiny, -fi.smallest_subnormal, -0.0, 0.0,
                     fi.smallest_subnormal, fi.tiny, 1.0, fi.max, np.inf], dtype=np.float32)
    rng = np.random.default_rng(0)
    more = np.sort(rng.standard_normal(5000).astype(np.float32) * 10.0 ** rng.uniform(-30, 30, 5000).astype(np.float32))
    for seq in (vals, more):
        k = _order_key(seq).astype(np.int64)
        assert np.all(np.diff(k) >= 0)
        strict = np.diff(seq.astype(np.float64)) > 0
        assert np.all(np.diff(k)[strict] > 0)                    # strictly increasing where the scores are
    assert _order_key(np.array([-0.0], np.float32))[0] == _order_key(np.array([0.0], np.float32))[0]
    nan = _order_key(np.array([np.nan], np.float32))[0]
    assert nan == 0 and np.all(_order_key(vals) > nan)            # NaN ranks below -inf
    # the inverse map (key_score) returns the score for every non-NaN key
    k = _order_key(vals)
    back = np.where(k & 0x80000000, k & 0x7FFFFFFF, ~k).astype(np.uint32).view(np.float32)
    assert np.array_equal(back, np.where(vals == 0, np.float32(0.0), vals))


def test_bf16_query_split_is_exact_down_to_2_pow_minus_41():
    """The score kernels split a bf16 query element x into hi = fp16(x) and
    lo = fp16((x - hi) * 2^24), the low part's products scaled back by 2^-24.  Replayed on
    every finite bf16 pattern in fp32 / fp16 (numpy rounds half to even, as cvt.rn):
    hi + lo * 2^-24 == x for every |x| >= 2^-41 inside fp16's range, and misses a smaller x
    by at most 2^-49."""
    bits = np.arange(1 << 16, dtype=np.uint32)
    x = (bits << 16).view(np.float32)
    fin = np.isfinite(x) & (np.abs(x) <= np.float32(65504.0))
    x = x[fin]
    with np.errstate(over="ignore"):
        hi = x.astype(np.float16).astype(np.float32)
        r = x - hi                                        # exact: hi is x rounded (or 0)
        lo = (r * np.float32(2.0 ** 24)).astype(np.float16).astype(np.float64)
    back = hi.astype(np.float64) + lo * 2.0 ** -24
    xd = x.astype(np.float64)
    big = np.abs(xd) >= 2.0 ** -41
    assert np.array_equal(back[big], xd[big])
    assert np.all(np.abs(back[~big] - xd[~big]) <= 2.0 ** -49)
    # without the 2^24 scale the residual of a small element is lost
    plain = hi.astype(np.float64) + (x - hi).astype(np.float16).astype(np.float64)
    assert not np.array_equal(plain[big], xd[big])
