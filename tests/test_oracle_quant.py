"""Pins of the oracle's block quantizers (BeeLLama.cpp v0.4.0 page, "Extended palette":
q2_0..q8_0 symmetric blocks, qb_1 blocks with a minimum; blocks of 32 with fp16 d)."""
import numpy as np
import pytest

import oracle

BITS = (2, 3, 4, 5, 6, 8)


def blocks(seed, n=400):
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((n, 32)) * np.exp2(rng.integers(-12, 12, (n, 1)))
    y[::17] *= 1e-6
    return y.astype(np.float32)


@pytest.mark.parametrize("bits", BITS)
def test_sym_round_trip_and_nearest_code(bits):
    qmax, qmin = 2 ** (bits - 1) - 1, -(2 ** (bits - 1))
    for y in blocks(bits):
        d16, codes = oracle.quant_sym(y, bits)
        # d = fp16(absmax / qmax), restated with numpy's IEEE float32 divide and fp16 cast
        ref_d = (np.float32(np.abs(y).max()) / np.float32(qmax)).astype(np.float16).view(np.uint16)
        assert d16 == ref_d
        d = float(oracle.f16_to_f32(np.array([d16], np.uint16))[0])
        assert codes.min() >= qmin and codes.max() <= qmax
        if d16 == 0:  # absmax/qmax rounds to zero in fp16: every code is 0
            assert not codes.any() and np.abs(y).max() / qmax <= 2.0**-25
            continue
        err = np.abs(y.astype(np.float64) - codes * d)
        if d16 >= 0x0400:  # normal fp16 d: absmax/d <= qmax + 0.5, no clamping
            assert np.all(err <= d / 2 * (1 + 2.0**-22))
        # brute force: the code is the nearest allowed value (exact ties excluded)
        cand = np.arange(qmin, qmax + 1)
        dist = np.abs(y.astype(np.float64)[:, None] - cand[None, :] * d)
        best = cand[np.argmin(dist, axis=1)]
        tie = np.sort(dist, axis=1)[:, 1] - np.sort(dist, axis=1)[:, 0] < 1e-9 * d
        assert np.array_equal(codes[~tie], best[~tie])


@pytest.mark.parametrize("bits", BITS)
def test_sym_zero_block_and_idempotence(bits):
    d16, codes = oracle.quant_sym(np.zeros(32, np.float32), bits)
    assert d16 == 0 and not codes.any()
    for y in blocks(bits + 10, 50):
        d16, codes = oracle.quant_sym(y, bits)
        d = oracle.f16_to_f32(np.array([d16], np.uint16))[0]
        d16b, codes2 = oracle.quant_sym((codes * d).astype(np.float32), bits)
        assert d16b == d16 and np.array_equal(codes2, codes)


@pytest.mark.parametrize("bits", (2, 3, 4, 5, 6))
def test_asym_round_trip(bits):
    qmax = 2**bits - 1
    rng = np.random.default_rng(bits)
    for _ in range(300):
        x = (rng.standard_normal(32) * rng.uniform(0.01, 10) + rng.uniform(-3, 3)).astype(np.float32)
        d16, m16, codes = oracle.quant_asym(x, bits)
        ref_d = ((np.float32(x.max()) - np.float32(x.min())) / np.float32(qmax)).astype(np.float16).view(np.uint16)
        assert d16 == ref_d
        assert m16 == np.float32(x.min()).astype(np.float16).view(np.uint16)
        d, m = (float(v) for v in oracle.f16_to_f32(np.array([d16, m16], np.uint16)))
        assert codes.min() >= 0 and codes.max() <= qmax
        err = np.abs(x.astype(np.float64) - (codes * d + m))
        assert np.all(err <= d / 2 * (1 + 2.0**-20) + abs(m - float(x.min())) + 1e-7 * abs(m))


def test_asym_constant_block_gives_zero_scale():
    d16, m16, codes = oracle.quant_asym(np.full(32, 1.5, np.float32), 4)
    assert d16 == 0 and not codes.any()
    assert oracle.f16_to_f32(np.array([m16], np.uint16))[0] == 1.5
