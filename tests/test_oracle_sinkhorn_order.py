"""Bit-exact pins of the oracle's kvarn arithmetic, restated here from the written definition.

What the pages fix ("Bonsai-Ternary-27B on 120k tokens", section "How the Walsh-Hadamard
transform and Sinkhorn save quality at 4-bit"; the KVarN section of the BeeLLama.cpp
v0.4.0 page): each head vector is rotated by the Walsh-Hadamard transform, then Sinkhorn
balancing picks a scale per channel and per token, then the balanced values are quantized.
The workload definition fixes the rest: 256-token groups, x -> H.x / sqrt(128) in a fixed
fp32 butterfly order, 8 iterations alternately dividing channels and tokens by their RMS,
fp16 scales, symmetric 4-bit blocks of 32.  What the pages leave open (and that decides
bits) is fixed by this build's reading, restated below in plain numpy from its text, not
from the oracle's code:

  * scale-only Sinkhorn: X2 = x*x; u_i = 1; each iteration computes the channel sums
    S_j = sum_i fma(X2_ij, u_i) and w_j = n / S_j, then the token sums
    R_i = sum_j fma(X2_ij, w_j) and u_i = 128 / R_i (a zero sum gives 1); after the last
    iteration c_j = sqrt(S_j / n) and t_i = sqrt(R_i / 128) (1 for a zero sum);
  * a channel sum is 32 partial sums: partial l is the fma chain (from 0, ascending) over
    the tokens l, l+64, l+128, l+192 plus the chain over l+32, l+96, l+160, l+224 (absent
    tokens of a partial group skipped); the partials are combined by an xor butterfly with
    offsets 16, 8, 4, 2, 1;
  * a token sum is 16 partial sums over runs of 8 consecutive channels (fma chains from 0,
    ascending), combined by an xor butterfly with offsets 8, 4, 2, 1;
  * the stored scales are fp16 (round to nearest even) clamped to [2^-14, 65504]; the
    balanced value is y = (x * (1/c16)) * (1/t16); blocks of 32 channels get
    d = fp16(absmax / qmax) (saturating) and code = clamp(rint(y / d), -2^(b-1), qmax).

Every fp32 operation is done by numpy on float32 arrays (IEEE, one rounding each); the
fused multiply-add, which numpy lacks, is computed exactly in float64 and rounded once
to fp32 (``fma32``, whose own pins are the first tests here).  The last test shows that
the inputs used can tell the written order apart from the plausible wrong ones (another
butterfly, another chain pairing, other channel runs, another recurrence).
"""
import fractions

import numpy as np
import pytest

import oracle

D = 128
GROUP = 256
KAPPA = np.array([0x3DB504F3], np.uint32).view(np.float32)[0]  # RN_fp32(2^-3.5)


# ---------------------------------------------------------------------------------------
# exact fp32 fused multiply-add

def fma32(a, b, c):
    """RN_fp32(a*b + c) for float32 arrays, with a single rounding.

    a*b is exact in float64 (24 + 24 significant bits); s = fl64(p + c) and its exact error
    e (two-sum) give p + c = s + e exactly.  Rounding s to fp32 is then the correct result
    except when s lies exactly halfway between two fp32 values and e != 0, where the sign of
    e decides."""
    a = np.asarray(a, np.float32)
    b = np.asarray(b, np.float32)
    c = np.asarray(c, np.float32)
    p = a.astype(np.float64) * b.astype(np.float64)
    c64 = c.astype(np.float64)
    s = p + c64
    bp = s - c64
    e = (p - bp) + (c64 - (s - bp))
    r = s.astype(np.float32)
    r64 = r.astype(np.float64)
    other = np.nextafter(r, np.where(s > r64, np.float32(np.inf), np.float32(-np.inf))).astype(np.float32)
    mid = (r64 + other.astype(np.float64)) * 0.5
    fix = (s != r64) & (s == mid) & (e != 0)
    toward_other = np.sign(e) == np.sign(other.astype(np.float64) - r64)
    return np.where(fix & toward_other, other, r).astype(np.float32)


def fma32_fraction(a, b, c):
    """The same operation on one triple by exact rational arithmetic (a slow second form)."""
    exact = fractions.Fraction(float(a)) * fractions.Fraction(float(b)) + fractions.Fraction(float(c))
    lo = np.float32(float(exact))  # within one fp32 step of the exact value
    cands = [np.nextafter(lo, np.float32(-np.inf)), lo, np.nextafter(lo, np.float32(np.inf))]
    dist = [abs(fractions.Fraction(float(x)) - exact) for x in cands]
    best = min(dist)
    winners = [x for x, dd in zip(cands, dist) if dd == best]
    if len(winners) == 1:
        return np.float32(winners[0])
    return np.float32([x for x in winners if (x.view(np.uint32) & 1) == 0][0])


def test_fma32_matches_exact_rational_rounding():
    rng = np.random.default_rng(0)
    a = (rng.standard_normal(3000) * np.exp2(rng.integers(-20, 20, 3000))).astype(np.float32)
    b = (rng.standard_normal(3000) * np.exp2(rng.integers(-20, 20, 3000))).astype(np.float32)
    c = (rng.standard_normal(3000) * np.exp2(rng.integers(-30, 30, 3000))).astype(np.float32)
    got = fma32(a, b, c)
    for i in range(3000):
        assert got[i] == fma32_fraction(a[i], b[i], c[i]), i


def test_fma32_rounds_halfway_cases_by_the_discarded_low_part():
    # 1 + 2^-24 is exactly halfway between 1 and 1 + 2^-23; a tiny extra term decides
    one = np.float32(1.0)
    half_ulp = np.float32(2.0**-24)
    assert fma32(half_ulp, one, one) == one  # tie -> even
    assert fma32(np.float32(1 + 2.0**-23), half_ulp, one) == np.float32(1 + 2.0**-23)  # just above
    assert fma32(np.float32(1 - 2.0**-24), half_ulp, one) == one  # just below
    # a product a*b that fp32 multiplication alone would round differently
    a = np.float32(1 + 2.0**-12)
    assert fma32(a, a, np.float32(-1.0)) == np.float32(2.0**-11 + 2.0**-24)


# ---------------------------------------------------------------------------------------
# the written definition of the scale-only Sinkhorn

def butterfly(p, offsets):
    """xor butterfly along axis 0: at each offset o, lane l takes p[l] + p[l ^ o]; returns
    lane 0 (every lane ends with the same value, fp32 addition being commutative)."""
    for o in offsets:
        idx = np.arange(p.shape[0]) ^ o
        p = (p + p[idx]).astype(np.float32)
    return p[0]


def channel_sums(x2, u, pairing="written"):
    """S_j for every channel j: 32 partials of two fma chains each, then the butterfly."""
    n = x2.shape[0]
    parts = np.zeros((32, D), np.float32)
    for l in range(32):
        if pairing == "halves":  # a plausible mistake: the two chains split the group in halves
            chains = ([l, l + 32, l + 64, l + 96], [l + 128, l + 160, l + 192, l + 224])
        else:
            chains = ([l, l + 64, l + 128, l + 192], [l + 32, l + 96, l + 160, l + 224])
        acc = []
        for chain in chains:
            a = np.zeros(D, np.float32)
            for i in chain:
                if i < n:
                    a = fma32(x2[i], np.full(D, u[i], np.float32), a)
            acc.append(a)
        parts[l] = (acc[0] + acc[1]).astype(np.float32)
    offs = (16, 8, 4, 2, 1) if pairing != "ascending" else (1, 2, 4, 8, 16)
    return butterfly(parts, offs)


def token_sums(x2, w, runs=16):
    """R_i for every token i: `runs` fma chains over consecutive channels, then the butterfly."""
    n = x2.shape[0]
    width = D // runs
    parts = np.zeros((runs, n), np.float32)
    for r in range(runs):
        a = np.zeros(n, np.float32)
        for j in range(width * r, width * r + width):
            a = fma32(x2[:, j], np.full(n, w[j], np.float32), a)
        parts[r] = a
    offs = tuple(runs >> k for k in range(1, runs.bit_length()))
    return butterfly(parts, offs)


def sinkhorn_written(x, iters=8, variant="written"):
    """Scales c (per channel) and t (per token) of one group by the written definition."""
    x = np.asarray(x, np.float32)
    n = x.shape[0]
    x2 = (x * x).astype(np.float32)
    fn = np.float32(n)
    u = np.ones(n, np.float32)
    S = np.zeros(D, np.float32)
    R = np.zeros(n, np.float32)
    for _ in range(iters):
        S = channel_sums(x2, u, "ascending" if variant == "ascending" else
                         ("halves" if variant == "halves" else "written"))
        w = np.where(S > 0, fn / np.where(S > 0, S, 1), np.float32(1)).astype(np.float32)
        if variant == "sqrt":  # another recurrence: carry c = sqrt(S/n) and take w = 1/(c*c)
            c = np.sqrt(np.where(S > 0, S / fn, 1).astype(np.float32))
            w = (np.float32(1) / (c * c)).astype(np.float32)
        R = token_sums(x2, w, 8 if variant == "runs8x16" else 16)
        u = np.where(R > 0, np.float32(128) / np.where(R > 0, R, 1), np.float32(1)).astype(np.float32)
    if iters == 0:
        return np.ones(D, np.float32), np.ones(n, np.float32)
    c = np.where(S > 0, np.sqrt((S / fn).astype(np.float32)), np.float32(1)).astype(np.float32)
    t = np.where(R > 0, np.sqrt((R / np.float32(128)).astype(np.float32)), np.float32(1)).astype(np.float32)
    return c, t


def group_tile(seed, n):
    """A rotated-looking group with spread channel and token scales (and a zero row when
    the group is long enough, which must get the scale 1)."""
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((n, D)) * np.exp(1.5 * rng.standard_normal(D))[None, :]
         * np.exp(0.7 * rng.standard_normal(n))[:, None])
    if n > 40:
        x[33] = 0.0
    return x.astype(np.float32)


@pytest.mark.parametrize("n", [1, 77, 255, 256])
def test_oracle_sinkhorn_is_the_written_order_bit_for_bit(n):
    x = group_tile(100 + n, n)
    for iters in (8, 3):
        c, t = oracle.sinkhorn(x, iters)
        cw, tw = sinkhorn_written(x, iters)
        assert np.array_equal(c.view(np.uint32), cw.view(np.uint32)), (n, iters)
        assert np.array_equal(t.view(np.uint32), tw.view(np.uint32)), (n, iters)


def test_written_order_is_distinguishable_from_plausible_mistakes():
    """Each variant is one plausible slip in the summation order or the recurrence; on the
    inputs of the test above each one changes at least one scale bit, so the bit-exact pin
    would catch it."""
    x = group_tile(356, 256)
    c, t = oracle.sinkhorn(x, 8)
    for variant in ("ascending", "halves", "runs8x16", "sqrt"):
        cv, tv = sinkhorn_written(x, 8, variant)
        same = np.array_equal(c.view(np.uint32), cv.view(np.uint32)) and np.array_equal(t.view(np.uint32),
                                                                                         tv.view(np.uint32))
        assert not same, variant


# ---------------------------------------------------------------------------------------
# the written kvarn composition: rotation, balancing, fp16 scales, normalization, blocks

def wht_written(x):
    """Rows of x (fp32) -> H.x.kappa: butterfly stages h = 1, 2, ..., 64 with
    (a, b) -> (a + b, a - b) on the pairs (i, i + h), i & h == 0, then one multiply."""
    v = np.array(x, np.float32, copy=True)
    h = 1
    while h < D:
        for i in range(D):
            if i & h:
                continue
            a, b = v[:, i].copy(), v[:, i + h].copy()
            v[:, i] = a + b
            v[:, i + h] = a - b
        h <<= 1
    return (v * KAPPA).astype(np.float32)


def f16_bits(x):
    return np.asarray(x, np.float32).astype(np.float16).view(np.uint16)


def f16_value(h):
    return np.asarray(h, np.uint16).view(np.float16).astype(np.float32)


def scale_bits(x):
    """fp16 of a positive scale, clamped to [2^-14, 65504]."""
    return np.clip(f16_bits(x), 0x0400, 0x7BFF).astype(np.uint16)


def block_quant(y, bits):
    """Symmetric blocks of 32 along the channels of each row: d16 [rows, 4], codes [rows, 128]."""
    qmax, qmin = 2 ** (bits - 1) - 1, -(2 ** (bits - 1))
    yb = y.reshape(-1, 4, 32)
    amax = np.abs(yb).max(axis=2).astype(np.float32)
    d16 = f16_bits((amax / np.float32(qmax)).astype(np.float32))
    d16 = np.where((d16 & 0x7FFF) == 0x7C00, (d16 & 0x8000) | 0x7BFF, d16).astype(np.uint16)
    df = f16_value(d16)
    safe = np.where(df != 0, df, np.float32(1))[:, :, None]
    q = np.rint((yb / safe).astype(np.float32))
    q = np.clip(q, qmin, qmax)
    q = np.where(df[:, :, None] != 0, q, 0)
    return d16, q.reshape(-1, D).astype(np.int16)


def kvarn_stream_written(xb, tail, bits, iters=8):
    """Quantized region of one kvarn stream from its BF16 rows, by the written definition:
    the oldest n - min(n, tail) tokens, in 256-token groups (the last one partial)."""
    n = xb.shape[0]
    Q = n - min(n, tail)
    x = (xb.astype(np.uint32) << 16).view(np.float32)
    codes = np.zeros((Q, D), np.int16)
    d16 = np.zeros((Q, 4), np.uint16)
    t16 = np.zeros(Q, np.uint16)
    c16 = np.zeros(((Q + GROUP - 1) // GROUP, D), np.uint16)
    for g0 in range(0, Q, GROUP):
        g1 = min(g0 + GROUP, Q)
        xr = wht_written(x[g0:g1])
        c, t = sinkhorn_written(xr, iters)
        ch = scale_bits(c)
        th = scale_bits(t)
        rc = (np.float32(1) / f16_value(ch)).astype(np.float32)
        rt = (np.float32(1) / f16_value(th)).astype(np.float32)
        y = ((xr * rc[None, :]).astype(np.float32) * rt[:, None]).astype(np.float32)
        dd, cc = block_quant(y, bits)
        codes[g0:g1], d16[g0:g1], t16[g0:g1], c16[g0 // GROUP] = cc, dd, th, ch
    return {"Q": Q, "codes": codes, "d16": d16, "t16": t16, "c16": c16}


def test_written_wht_is_the_oracle_rotation():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal((40, D)) * np.exp(rng.standard_normal(D))).astype(np.float32)
    assert np.array_equal(wht_written(x).view(np.uint32), oracle.wht128(x).view(np.uint32))


@pytest.mark.parametrize("kind", ["kvarn2", "kvarn3", "kvarn4", "kvarn5", "kvarn6", "kvarn8"])
def test_oracle_kvarn_stream_is_the_written_composition(kind):
    """A 300-token stream with a 20-token tail: one full group and a partial one of 24."""
    bits = int(kind[-1])
    rng = np.random.default_rng(bits)
    k = rng.standard_normal((300, D)) * np.exp(0.5 * rng.standard_normal(D))[None, :]
    k[:, [5, 70]] *= 20.0
    xb = (np.ascontiguousarray(k, np.float32).view(np.uint32) + 0x7FFF
          + ((np.ascontiguousarray(k, np.float32).view(np.uint32) >> 16) & 1)) >> 16
    xb = xb.astype(np.uint16)
    st = oracle.stream_state(kind, xb, 20)
    ref = kvarn_stream_written(xb, 20, bits)
    assert st["Q"] == ref["Q"] == 280
    for key in ("codes", "d16", "t16", "c16"):
        assert np.array_equal(st[key], ref[key]), key
