"""Pins of the oracle's Sinkhorn balancing (Bonsai-Ternary-27B page, "How the WHT and
Sinkhorn save quality": a per-dimension scale equalizes the spread before quantizing;
the steps used are 8 iterations of channel-RMS then token-RMS division into fp16 scales)."""
import numpy as np

import oracle

D = 128


def literal_numpy(x, iters):
    """Independent restatement: divide channels by their RMS over tokens, then tokens by
    their RMS over channels, accumulating the divisors."""
    y = x.astype(np.float64).copy()
    c = np.ones(D)
    t = np.ones(x.shape[0])
    for _ in range(iters):
        r = np.sqrt(np.mean(y * y, axis=0))
        y /= r[None, :]
        c *= r
        r = np.sqrt(np.mean(y * y, axis=1))
        y /= r[:, None]
        t *= r
    return c, t


def tile(seed, n=256):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, D)) * np.exp(rng.standard_normal(D))[None, :] * np.exp(0.5 * rng.standard_normal(n))[:, None]
    return x.astype(np.float32)


def test_scale_only_form_matches_literal_forms():
    for seed, n in ((0, 256), (1, 77), (2, 1), (3, 255)):
        x = tile(seed, n)
        c, t = oracle.sinkhorn(x, 8)
        cl, tl = oracle.sinkhorn_literal(x.astype(np.float64), 8)
        cn, tn = literal_numpy(x, 8)
        for a, b in ((c, cl), (c, cn), (cl, cn)):
            assert np.max(np.abs(a / b - 1)) < 1e-5
        for a, b in ((t, tl), (t, tn)):
            assert np.max(np.abs(a / b - 1)) < 1e-5


def test_token_rms_is_one_after_last_step():
    x = tile(4)
    c, t = oracle.sinkhorn(x, 8)
    y = x.astype(np.float64) / (c[None, :].astype(np.float64) * t[:, None].astype(np.float64))
    assert np.max(np.abs(np.sqrt(np.mean(y * y, axis=1)) - 1)) < 1e-5
    # the channel RMS converges towards 1 as well
    assert np.max(np.abs(np.sqrt(np.mean(y * y, axis=0)) - 1)) < 0.05


def test_rank_one_magnitudes_converge_in_one_iteration():
    rng = np.random.default_rng(5)
    n = 256
    alpha = np.exp(rng.uniform(-2, 2, n))
    beta = np.exp(rng.uniform(-2, 2, D))
    sigma = rng.choice([-1.0, 1.0], (n, D))
    x = (alpha[:, None] * beta[None, :] * sigma).astype(np.float32)
    c, t = oracle.sinkhorn(x, 1)
    y = x.astype(np.float64) / (c[None, :] * t[:, None])
    assert np.max(np.abs(np.abs(y) - 1)) < 1e-5
    # closed form of the quantized result: every code is sign * qmax
    c16 = oracle.f32_to_f16(c)
    t16 = oracle.f32_to_f16(t)
    rc = np.float32(1) / oracle.f16_to_f32(c16)
    rt = np.float32(1) / oracle.f16_to_f32(t16)
    yq = (x * rc[None, :]) * rt[:, None]
    for bits in (2, 3, 4, 5, 6, 8):
        qmax = 2 ** (bits - 1) - 1
        for i in (0, 100, 255):
            for b in range(4):
                _, codes = oracle.quant_sym(yq[i, 32 * b:32 * b + 32], bits)
                assert np.array_equal(codes, (sigma[i, 32 * b:32 * b + 32] * qmax).astype(np.int16))


def test_zero_channel_and_token_get_unit_scale():
    x = tile(6, 64)
    x[:, 5] = 0
    x[9, :] = 0
    c, t = oracle.sinkhorn(x, 8)
    assert c[5] == 1.0 and t[9] == 1.0
    assert np.all(np.isfinite(c)) and np.all(np.isfinite(t))
