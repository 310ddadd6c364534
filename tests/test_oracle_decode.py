"""Pins of the oracle's stream state and fp64 decode reference.

Tail rule (BeeLLama.cpp v0.4.0 page, "KV Cache Precision Tail": the newest N tokens stay
16-bit, positions 0..n-N-1 are stored in the low-bit type) and the kvarn group rule; the
decode reference equals textbook softmax attention when nothing is quantized."""
import numpy as np
import pytest

import oracle
from bit_kv_cache_17_b200 import synth

D = 128


def textbook_attention(q, k, v, scale):
    s = (q.astype(np.float64) @ k.astype(np.float64).T) * scale
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    return p @ v.astype(np.float64)


def test_pure_bf16_equals_textbook_attention():
    rng = np.random.default_rng(0)
    for n, G in ((1, 1), (5, 3), (300, 4)):
        k = synth.bf16_bits(rng.standard_normal((n, D)).astype(np.float32))
        v = synth.bf16_bits(rng.standard_normal((n, D)).astype(np.float32))
        q = rng.standard_normal((G, D)).astype(np.float32)
        scale = 1 / np.sqrt(D)
        for t in ("bf16", "kvarn4", "q4_0"):
            out = oracle.decode_head(t, t, k, v, tail=n if t != "bf16" else 0, q=q)
            ref = textbook_attention(q, synth.bf16_to_f32(k), synth.bf16_to_f32(v), scale)
            assert np.max(np.abs(out - ref)) < 1e-12


def test_tail_rule_and_state_sizes():
    rng = np.random.default_rng(1)
    x = synth.bf16_bits(rng.standard_normal((700, D)).astype(np.float32))
    for tail in (0, 1, 255, 256, 699, 700, 5000):
        for t in ("q3_0", "kvarn2", "q4_1"):
            st = oracle.stream_state(t, x, tail)
            assert st["Q"] == 700 - min(700, tail)
            assert st["codes"].shape == (st["Q"], D)
            assert st["c16"].shape == ((st["Q"] + 255) // 256, D)


def test_full_groups_are_final_and_partial_groups_follow_their_rows():
    rng = np.random.default_rng(2)
    x = synth.bf16_bits(rng.standard_normal((900, D)).astype(np.float32))
    a = oracle.stream_state("kvarn4", x[:600], 0)   # groups [0,256) [256,512) full, [512,600) partial
    b = oracle.stream_state("kvarn4", x[:900], 0)   # group [512,768) full now
    assert np.array_equal(a["codes"][:512], b["codes"][:512])
    assert np.array_equal(a["c16"][:2], b["c16"][:2])
    # the partial group is a function of its own rows only
    c = oracle.stream_state("kvarn4", x[512:600], 0)
    assert np.array_equal(a["codes"][512:600], c["codes"])
    assert np.array_equal(a["c16"][2], c["c16"][0])
    # qb types quantize tokens independently
    qa = oracle.stream_state("q5_0", x[:600], 0)
    qb = oracle.stream_state("q5_0", x[:900], 0)
    assert np.array_equal(qa["codes"], qb["codes"][:600])


def test_one_hot_query_returns_that_value_row():
    rng = np.random.default_rng(3)
    n = 600
    k = synth.bf16_bits(rng.standard_normal((n, D)).astype(np.float32))
    v = synth.bf16_bits(rng.standard_normal((n, D)).astype(np.float32))
    for t, tail in (("kvarn4", 64), ("q4_0", 0), ("q4_1", 10)):
        st = oracle.stream_state(t, k, tail)
        kd = np.concatenate([oracle.dequant(t, st), synth.bf16_to_f32(k[st["Q"]:]).astype(np.float64)])
        vs = oracle.stream_state(t, v, tail)
        vd = np.concatenate([oracle.dequant(t, vs), synth.bf16_to_f32(v[vs["Q"]:]).astype(np.float64)])
        i = int(np.argmax(np.linalg.norm(kd, axis=1)))
        q = (kd[i] / np.linalg.norm(kd[i]) * 1e4).astype(np.float32)[None, :]
        out = oracle.decode_head(t, t, k, v, tail, q)
        assert np.max(np.abs(out[0] - vd[i])) < 1e-6 * np.abs(vd[i]).max()


@pytest.mark.parametrize("t", ["kvarn4", "q2_0", "q6_1"])
def test_constant_values_come_back(t):
    rng = np.random.default_rng(4)
    n = 520
    k = synth.bf16_bits(rng.standard_normal((n, D)).astype(np.float32))
    row = synth.bf16_bits(np.linspace(-2, 2, D).astype(np.float32))
    v = np.tile(row, (n, 1))
    q = rng.standard_normal((3, D)).astype(np.float32)
    out = oracle.decode_head(t, t, k, v, 100, q)
    vs = oracle.stream_state(t, v, 100)
    vrow = oracle.dequant(t, vs)[0]
    # quantized rows are all equal to vrow (same input, same scales); tail rows are exact
    assert np.allclose(oracle.dequant(t, vs), vrow[None, :], atol=0)
    lo = np.minimum(vrow, synth.bf16_to_f32(row))
    hi = np.maximum(vrow, synth.bf16_to_f32(row))
    assert np.all(out >= lo - 1e-12) and np.all(out <= hi + 1e-12)


def test_dequant_rotated_basis_is_rotation_of_original():
    rng = np.random.default_rng(5)
    x = synth.bf16_bits(rng.standard_normal((300, D)).astype(np.float32))
    st = oracle.stream_state("kvarn5", x, 20)
    a = oracle.dequant("kvarn5", st, basis=0)
    b = oracle.dequant("kvarn5", st, basis=1)
    assert np.allclose(oracle.wht128_f64(b), a, atol=1e-12)
    # and the rotation undoes the forward one up to quantization error
    xr = synth.bf16_to_f32(x[:280]).astype(np.float64)
    rel = np.linalg.norm(a - xr) / np.linalg.norm(xr)
    assert rel < 0.1


def test_prefill_chunk_reduces_to_decode_and_to_masked_attention():
    """The chunk reference (query i of the n_q newest tokens sees the first n - n_q + 1 + i
    rows of the full history's state): with one query it is the decode reference; with BF16
    rows it is textbook causal attention; with quantized rows it is textbook attention over
    the prefix of the dequantized state (positions >= Q exact BF16)."""
    rng = np.random.default_rng(5)
    n, G, n_q, tail = 700, 3, 9, 200
    k, v, _ = synth.kv_ar1(rng, 1, n)
    k, v = k[0], v[0]
    q = rng.standard_normal((n_q, G, D)).astype(np.float32)
    scale = 1 / np.sqrt(D)
    for t in ("kvarn4", "q4_0", "q3_1", "bf16"):
        tl = tail if t != "bf16" else 0
        out = oracle.prefill_head(t, t, k, v, tl, q)
        one = oracle.prefill_head(t, t, k, v, tl, q[-1:])
        assert np.array_equal(one[0], oracle.decode_head(t, t, k, v, tl, q[-1]))
        assert np.array_equal(out[-1], one[0])
        if t == "bf16":
            kf, vf = synth.bf16_to_f32(k), synth.bf16_to_f32(v)
        else:
            st_k, st_v = oracle.stream_state(t, k, tl), oracle.stream_state(t, v, tl)
            Q = st_k["Q"]
            kf = np.concatenate([oracle.dequant(t, st_k), synth.bf16_to_f32(k[Q:])])
            vf = np.concatenate([oracle.dequant(t, st_v), synth.bf16_to_f32(v[Q:])])
        for i in range(n_q):
            ni = n - n_q + 1 + i
            ref = textbook_attention(q[i], kf[:ni], vf[:ni], scale)
            assert np.max(np.abs(out[i] - ref)) < 1e-10, (t, i)


def test_mixed_types_reduce_to_closed_forms():
    """K and V of different types: the K stream only decides the weights, the V stream only the
    values.  With every token quantized (tail 0) and a q type, whose tokens are quantized one by
    one, identical input rows give identical stored rows.  Constant keys then give equal
    weights, so the output is the mean of the V type's dequantized rows; constant values give
    that one row whatever the weights."""
    rng = np.random.default_rng(5)
    n, G = 700, 3
    q = rng.standard_normal((G, D)).astype(np.float32)
    const = np.tile(synth.bf16_bits(rng.standard_normal((1, D)).astype(np.float32)), (n, 1))
    for tk, tv in (("q8_0", "kvarn2"), ("q4_1", "q3_0"), ("q5_0", "kvarn4")):
        v = synth.bf16_bits(rng.standard_normal((n, D)).astype(np.float32))
        out = oracle.decode_head(tk, tv, const, v, 0, q)
        rows = oracle.dequant(tv, oracle.stream_state(tv, v, 0))
        assert np.max(np.abs(out - rows.mean(axis=0)[None, :])) < 1e-12
    for tk, tv in (("kvarn4", "q3_0"), ("kvarn2", "q6_1"), ("q8_0", "q2_0")):
        k = synth.bf16_bits(rng.standard_normal((n, D)).astype(np.float32))
        out = oracle.decode_head(tk, tv, k, const, 0, q)
        rows = oracle.dequant(tv, oracle.stream_state(tv, const, 0))
        assert np.array_equal(rows, np.tile(rows[:1], (n, 1)))
        assert np.max(np.abs(out - rows[:1])) < 1e-12
