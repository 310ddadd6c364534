"""K and V of different types (the pages' separate --cache-type-k / --cache-type-v switches)
and the --cache-var-norm switch, against the CPU oracle.

Mixed types decode with two kernels: Q.K of the K type writes the scores of the quantized
prefix to the workspace, softmax and P.V of the V type read them.  Every packed byte of both
streams equals the oracle's state of its own type; the decode, the one-step append + decode
and the chunk attention agree with the oracle's fp64 attention over the two dequantized
streams (relative L2 <= 1e-3, max abs <= 2e-3 x RMS)."""
import numpy as np
import pytest

import gpu_helpers as H
import oracle
from bit_kv_cache_17_b200 import kvq, synth

pytestmark = pytest.mark.gpu

PAIRS = [("kvarn4", "q3_0"), ("q8_0", "q4_0"), ("q4_1", "kvarn2"), ("kvarn3", "q5_1"), ("q2_0", "kvarn8")]


def _rows(x, a, b):
    return synth.token_major(x[:, a:b])


def _decode_ref(tk, tv, k, v, n, tail, q, hkv):
    G = q.shape[0] // hkv
    out = np.zeros((q.shape[0], 128))
    for h in range(hkv):
        out[h * G:(h + 1) * G] = oracle.decode_head(tk, tv, k[h, :n], v[h, :n], tail, q[h * G:(h + 1) * G])
    return out


@pytest.mark.parametrize("tk,tv", PAIRS)
def test_mixed_types_decode(tk, tv):
    """Sequences inside the tail (no quantized prefix), with a partial kvarn group, and several
    groups long; GQA 5."""
    th = H.torch()
    hkv, hq, tail = 2, 10, 100
    lens = [60, 100 + 256 + 70, 100 + 3 * 256 + 5, 1500]
    rng = np.random.default_rng(7)
    data = [synth.kv_ar1(rng, hkv, n)[:2] for n in lens]
    c = H.make_cache(tk, hkv, 2048, tail, n_seqs=len(lens), type_v=tv)
    H.append(c, 0, list(range(len(lens))), [(_rows(d[0], 0, n), _rows(d[1], 0, n)) for d, n in zip(data, lens)])
    q = synth.queries(rng, 1, len(lens), hq)[0]
    ids = [2, 0, 3, 1]
    out = c.decode(0, ids, th.from_numpy(q[ids]).cuda())
    th.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    buf = H.storage_bytes(c)
    for row, s in enumerate(ids):
        k, v = data[s]
        for h in range(hkv):
            H.compare_stream(c, buf, tk, 0, s, h, 0, k[h], tail)
            H.compare_stream(c, buf, tv, 0, s, h, 1, v[h], tail)
        ref = _decode_ref(tk, tv, k, v, lens[s], tail, q[s], hkv)
        H.check_decode(got[row], ref, f"{tk}/{tv} seq {s}")
    assert c.status() == 0


def test_mixed_types_append_decode_steps():
    """One-token steps (spills into the quantized groups of both types) through the fused step
    entry point, which runs its decode after the append in stream order for mixed types."""
    th = H.torch()
    tk, tv = "kvarn4", "q3_0"
    hkv, hq, tail = 2, 8, 64
    rng = np.random.default_rng(11)
    n = 64 + 256 - 2
    k, v, _ = synth.kv_ar1(rng, hkv, n + 6)
    c = H.make_cache(tk, hkv, 1024, tail, type_v=tv)
    H.append(c, 0, [0], [(_rows(k, 0, n), _rows(v, 0, n))])
    for step in range(6):
        q = synth.queries(rng, 1, 1, hq)[0]
        out = c.append_decode(0, [0], [1], H.to_dev_bf16(_rows(k, n, n + 1)), H.to_dev_bf16(_rows(v, n, n + 1)),
                              th.from_numpy(q).cuda())
        th.cuda.synchronize()
        n += 1
        buf = H.storage_bytes(c)
        for h in range(hkv):
            H.compare_stream(c, buf, tk, 0, 0, h, 0, k[h, :n], tail)
            H.compare_stream(c, buf, tv, 0, 0, h, 1, v[h, :n], tail)
        H.check_decode(out.cpu().numpy()[0].astype(np.float64), _decode_ref(tk, tv, k, v, n, tail, q[0], hkv),
                       f"step {step}")
    assert c.status() == 0


def test_mixed_types_prefill_chunk():
    th = H.torch()
    tk, tv = "q8_0", "kvarn3"
    hkv, G, tail, n, n_q = 2, 4, 128, 900, 80
    rng = np.random.default_rng(13)
    k, v, _ = synth.kv_ar1(rng, hkv, n)
    c = H.make_cache(tk, hkv, 1024, tail, type_v=tv)
    H.append(c, 0, [0], [(_rows(k, 0, n), _rows(v, 0, n))])
    q = rng.standard_normal((n_q, hkv * G, 128)).astype(np.float32)
    out = c.prefill_attn(0, 0, th.from_numpy(q).cuda())
    th.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    for h in range(hkv):
        ref = oracle.prefill_head(tk, tv, k[h], v[h], tail, q[:, h * G:(h + 1) * G])
        for i in range(n_q):
            H.check_decode(got[i, h * G:(h + 1) * G], ref[i], f"head {h} query {i}")
    assert c.status() == 0


def test_mixed_types_workspace_holds_the_scores():
    c = H.make_cache("kvarn4", 2, 1000, 64, n_seqs=3, type_v="q3_0")
    same = H.make_cache("kvarn4", 2, 1000, 64, n_seqs=3)
    extra = kvq.kvq_workspace_bytes(c.handle, 3, 10) - kvq.kvq_workspace_bytes(same.handle, 3, 10)
    assert extra == 4 * 3 * 10 * 1024


@pytest.mark.parametrize("tq,tkv", [("q4_0", "kvarn4"), ("q2_0", "kvarn2")])
def test_var_norm_cache_is_the_kvarn_cache(tq, tkv):
    """qN_0 with var_norm = 1 stores and decodes exactly as kvarnN."""
    th = H.torch()
    from bit_kv_cache_17_b200.kvq import KVCache

    hkv, hq, tail, n = 2, 6, 100, 700
    rng = np.random.default_rng(17)
    k, v, _ = synth.kv_ar1(rng, hkv, n)
    c = KVCache(n_layers=1, n_seqs=1, n_kv_heads=hkv, max_ctx=1024, type_k=tq, type_v=tq, tail=tail, var_norm=1)
    H.append(c, 0, [0], [(_rows(k, 0, n), _rows(v, 0, n))])
    q = synth.queries(rng, 1, 1, hq)[0]
    out = c.decode(0, [0], th.from_numpy(q).cuda())
    th.cuda.synchronize()
    buf = H.storage_bytes(c)
    for h in range(hkv):
        H.compare_stream(c, buf, tkv, 0, 0, h, 0, k[h], tail)
        H.compare_stream(c, buf, tkv, 0, 0, h, 1, v[h], tail)
    H.check_decode(out.cpu().numpy()[0].astype(np.float64), _decode_ref(tkv, tkv, k, v, n, tail, q[0], hkv), tq)
    assert c.status() == 0
