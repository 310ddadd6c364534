"""Pins of the oracle's number formats (round to nearest, ties to even).

fp16: numpy's float32 -> float16 cast (IEEE round to nearest even) is the library
routine the oracle's hand-written conversion must reproduce bit for bit.
bf16: brute force nearest of the two bracketing BF16 values, computed in float64.
"""
import numpy as np

import oracle


def _sample_f32_bits(n, seed):
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 2**32, n, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    return x[np.isfinite(x)]


def test_f16_matches_numpy_cast():
    specials = np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 65536.0, 1e9, 2.0**-14, 2.0**-24,
                         2.0**-25, 3 * 2.0**-26, 2.0**-25 * 1.0000001, 5.960464477539063e-08,
                         6.097555160522461e-05, 1.0 + 2.0**-11, 1.0 + 3 * 2.0**-11, -2.5e-6],
                        dtype=np.float32)
    rng = np.random.default_rng(5)
    ranged = (rng.standard_normal(200000) * np.exp2(rng.uniform(-30, 17, 200000))).astype(np.float32)
    for x in (specials, _sample_f32_bits(200000, 1), ranged):
        with np.errstate(over="ignore"):
            ref = x.astype(np.float16).view(np.uint16)
        got = oracle.f32_to_f16(x)
        assert np.array_equal(got, ref)


def test_f16_to_f32_exhaustive():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = h.view(np.float16).astype(np.float32)
    got = oracle.f16_to_f32(h)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_bf16_is_nearest_even():
    x = np.concatenate([_sample_f32_bits(100000, 2),
                        np.random.default_rng(3).standard_normal(100000).astype(np.float32)])
    x = x[np.abs(x) < 3e38]
    got = oracle.f32_to_bf16(x)
    u = x.view(np.uint32)
    lo = (u >> 16).astype(np.uint32)
    hi = lo + 1
    vlo = (lo << 16).view(np.float32).astype(np.float64)
    vhi = (hi << 16).view(np.float32).astype(np.float64)
    xd = x.astype(np.float64)
    dlo, dhi = np.abs(xd - vlo), np.abs(vhi - xd)
    pick_hi = (dhi < dlo) | ((dhi == dlo) & ((lo & 1) == 1))
    ref = np.where(pick_hi, hi, lo).astype(np.uint16)
    assert np.array_equal(got, ref)


def test_every_f16_rounding_of_a_bf16_value_is_a_bf16_value():
    """The F16 tail reading rests on this: fp16(x) of any BF16 x (all 65 536 patterns, NaN
    aside) is exactly representable in BF16, so a stream with an F16 tail equals the BF16-tail
    stream of the rounded rows.  The fp16 cast here is numpy's, independent of the oracle."""
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    x = (h.astype(np.uint32) << 16).view(np.float32)
    y = x.astype(np.float16).astype(np.float32)  # IEEE round to nearest even, overflow to inf
    ok = ~np.isnan(x)
    back = ((y.view(np.uint32) >> 16) << 16).view(np.float32)  # truncation to BF16 loses nothing
    assert np.array_equal(back[ok], y[ok])
    # the oracle's helper agrees with numpy, and changes only out-of-range values
    rows = oracle.f16_tail_rows(h[ok])
    assert np.array_equal(oracle.bf16_to_f32(rows), y[ok])
    moved = np.nonzero(oracle.bf16_to_f32(rows) != x[ok])[0]
    ax = np.abs(x[ok][moved])
    assert np.all((ax < 2.0**-14) | (ax > 65504.0))
    assert np.array_equal(oracle.f16_tail_bits(h[ok]), x[ok].astype(np.float16).view(np.uint16))
