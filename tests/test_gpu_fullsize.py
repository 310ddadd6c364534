"""Parity at the workloads' full sizes, in the launch configuration bench.py times (a long
prefill, then one-token appends, then decode).  Every packed byte of the sampled streams is
compared with the oracle, and the decode output of sampled KV heads (the oracle decodes one
KV head at a time from its full BF16 history).

Workloads: decode at 64k context (kvarn2..kvarn8, 8 KV heads, 40 query heads, tail 1024);
plain block formats at 16k (tails 0, 1024, 2048); 16 sequences of 4096..32768 tokens with a
4096-token batched append and batched decode; one layer of the 240k-token shape (kvarn2,
q4_0 with tail 1024, BF16)."""
import numpy as np
import pytest

import gpu_helpers as H
from bit_kv_cache_17_b200 import synth

pytestmark = pytest.mark.gpu


def _dev(bits):
    return H.to_dev_bf16(bits)


def _check_heads(cache, type_, layer, seq, k, v, tail, heads, q=None, n_q_heads=None, out=None):
    buf = H.storage_bytes(cache)
    for h in heads:
        H.compare_stream(cache, buf, type_, layer, seq, h, 0, k[h], tail)
        H.compare_stream(cache, buf, type_, layer, seq, h, 1, v[h], tail)
    if q is not None:
        hkv = k.shape[0]
        G = n_q_heads // hkv
        for h in heads:
            import oracle

            ref = oracle.decode_head(type_, type_, k[h], v[h], tail if type_ != "bf16" else 0, q[h * G:(h + 1) * G])
            H.check_decode(out[h * G:(h + 1) * G], ref, f"{type_} head {h}")


@pytest.fixture(scope="module")
def cfg2():
    return synth.config2()


@pytest.mark.parametrize("t", ["kvarn2", "kvarn3", "kvarn4", "kvarn5", "kvarn6", "kvarn8"])
def test_decode_64k(cfg2, t):
    th = H.torch()
    n, hkv, hq, tail = cfg2["n"], cfg2["hkv"], cfg2["hq"], cfg2["tail"]
    c = H.make_cache(t, hkv, n, tail)
    kt, vt = _dev(synth.token_major(cfg2["k"])), _dev(synth.token_major(cfg2["v"]))
    P = n - 3
    c.append(0, [0], [P], kt[:P], vt[:P])
    for i in range(3):  # one-token steps, the last one at context 65536
        c.append(0, [0], [1], kt[P + i:P + i + 1], vt[P + i:P + i + 1])
    q = cfg2["q"][0, 0]
    out = c.decode(0, [0], th.from_numpy(q).cuda()[None])
    th.cuda.synchronize()
    _check_heads(c, t, 0, 0, cfg2["k"], cfg2["v"], tail, [0, 5], q, hq, out.cpu().numpy()[0].astype(np.float64))
    assert c.status() == 0


@pytest.fixture(scope="module")
def cfg1():
    return synth.config1()


@pytest.mark.parametrize("tail", [0, 1024, 2048])
@pytest.mark.parametrize("t", ["q2_0", "q3_0", "q4_0", "q5_0", "q6_0", "q8_0", "q4_1"])
def test_formats_16k(cfg1, t, tail):
    th = H.torch()
    n, hkv, hq = cfg1["n"], cfg1["hkv"], cfg1["hq"]
    c = H.make_cache(t, hkv, n, tail)
    kt, vt = _dev(synth.token_major(cfg1["k"])), _dev(synth.token_major(cfg1["v"]))
    c.append(0, [0], [n - 1], kt[:n - 1], vt[:n - 1])
    c.append(0, [0], [1], kt[n - 1:], vt[n - 1:])
    q = cfg1["q"][0, 0]
    out = c.decode(0, [0], th.from_numpy(q).cuda()[None])
    th.cuda.synchronize()
    _check_heads(c, t, 0, 0, cfg1["k"], cfg1["v"], tail, [3], q, hq, out.cpu().numpy()[0].astype(np.float64))


def test_batched_16_sequences():
    th = H.torch()
    cfg = synth.config3(steps=2)
    hkv, hq, tail, P = cfg["hkv"], cfg["hq"], cfg["tail"], cfg["prefill"]
    Ls = cfg["lengths"]
    S = len(Ls)
    c = H.make_cache("kvarn4", hkv, max(Ls) + P + 2, tail, n_seqs=S)
    ks = [_dev(synth.token_major(k)) for k in cfg["k"]]
    vs = [_dev(synth.token_major(v)) for v in cfg["v"]]
    c.append(0, list(range(S)), Ls, th.cat([k[:l] for k, l in zip(ks, Ls)]), th.cat([v[:l] for v, l in zip(vs, Ls)]))
    c.append(0, list(range(S)), [P] * S, th.cat([k[l:l + P] for k, l in zip(ks, Ls)]),
             th.cat([v[l:l + P] for v, l in zip(vs, Ls)]))
    for step in range(2):
        off = [l + P + step for l in Ls]
        c.append(0, list(range(S)), [1] * S, th.cat([k[o:o + 1] for k, o in zip(ks, off)]),
                 th.cat([v[o:o + 1] for v, o in zip(vs, off)]))
        out = c.decode(0, list(range(S)), th.from_numpy(cfg["q"][step]).cuda())
    th.cuda.synchronize()
    out = out.cpu().numpy().astype(np.float64)
    for s in (0, 7, 15):
        n = Ls[s] + P + 2
        k, v = cfg["k"][s][:, :n], cfg["v"][s][:, :n]
        buf = H.storage_bytes(c)
        H.compare_stream(c, buf, "kvarn4", 0, s, 2, 0, k[2], tail)
        H.compare_stream(c, buf, "kvarn4", 0, s, 2, 1, v[2], tail)
        import oracle

        G = hq // hkv
        ref = oracle.decode_head("kvarn4", "kvarn4", k[2], v[2], tail, cfg["q"][1, s, 2 * G:3 * G])
        H.check_decode(out[s, 2 * G:3 * G], ref, f"seq {s}")


@pytest.fixture(scope="module")
def cfg4():
    return synth.config4_layer(7)


@pytest.mark.parametrize("t", ["kvarn2", "q4_0", "bf16"])
def test_layer_240k(cfg4, t):
    th = H.torch()
    n, hkv, hq, tail = cfg4["n"], cfg4["hkv"], cfg4["hq"], cfg4["tail"]
    c = H.make_cache(t, hkv, n, tail)
    kt, vt = _dev(synth.token_major(cfg4["k"])), _dev(synth.token_major(cfg4["v"]))
    c.append(0, [0], [n - 1], kt[:n - 1], vt[:n - 1])
    c.append(0, [0], [1], kt[n - 1:], vt[n - 1:])
    q = cfg4["q"][0, 0]
    out = c.decode(0, [0], th.from_numpy(q).cuda()[None])
    th.cuda.synchronize()
    _check_heads(c, t, 0, 0, cfg4["k"], cfg4["v"], tail, [6], q, hq, out.cpu().numpy()[0].astype(np.float64))


def test_zero_and_constant_rows_quantize_like_the_oracle():
    hkv, tail = 1, 16
    n = 600
    k = np.zeros((hkv, n, 128), np.uint16)
    v = np.tile(synth.bf16_bits(np.linspace(-3, 3, 128).astype(np.float32)), (hkv, n, 1))
    k[:, 300:] = synth.bf16_bits(np.random.default_rng(0).standard_normal((hkv, n - 300, 128)).astype(np.float32))
    for t in ("kvarn4", "q3_0", "q5_1"):
        c = H.make_cache(t, hkv, 1024, tail)
        H.append(c, 0, [0], [(synth.token_major(k), synth.token_major(v))])
        buf = H.storage_bytes(c)
        H.compare_stream(c, buf, t, 0, 0, 0, 0, k[0], tail)
        H.compare_stream(c, buf, t, 0, 0, 0, 1, v[0], tail)
