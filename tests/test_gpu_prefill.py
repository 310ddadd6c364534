"""kvq_prefill_attn (a chunk of queries, causal over the chunk's own tokens) against the CPU
oracle's chunk reference: query i sees the first n - n_q + 1 + i tokens of the cache state
of the full history (relative L2 <= 1e-3, max abs <= 2e-3 x RMS per query row).

Cases: a chunk inside the BF16 tail; a chunk longer than the tail (the early queries end
inside the quantized prefix); more than 16 queries (several launches); GQA 5; the BF16 type;
chunks of 64 and 256 queries at context 65536; every quantized type; caches with an F16 tail."""
import numpy as np
import pytest

import gpu_helpers as H
import oracle
from bit_kv_cache_17_b200 import kvq, synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("type_,n,n_q,tail", [("kvarn4", 1524, 24, 200), ("q4_0", 1524, 300, 200),
                                              ("kvarn2", 900, 70, 64), ("bf16", 600, 40, 0),
                                              ("q8_0", 333, 333, 1000)])
def test_prefill_chunk_matches_oracle(type_, n, n_q, tail):
    th = H.torch()
    hkv, G = 2, 5
    rng = np.random.default_rng(n + n_q)
    k, v, _ = synth.kv_ar1(rng, hkv, n)
    c = H.make_cache(type_, hkv, 2048, tail)
    H.append(c, 0, [0], [(synth.token_major(k), synth.token_major(v))])
    q = rng.standard_normal((n_q, hkv * G, 128)).astype(np.float32)
    out = c.prefill_attn(0, 0, th.from_numpy(q).cuda())
    th.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    for h in range(hkv):
        ref = oracle.prefill_head(type_, type_, k[h], v[h], tail, q[:, h * G:(h + 1) * G])
        for i in range(n_q):
            H.check_decode(got[i, h * G:(h + 1) * G], ref[i], f"{type_} head {h} query {i}")
    assert c.status() == 0


def test_prefill_rejects_a_chunk_longer_than_the_sequence():
    th = H.torch()
    c = H.make_cache("q4_0", 1, 512, 64)
    rng = np.random.default_rng(3)
    k, v, _ = synth.kv_ar1(rng, 1, 10)
    H.append(c, 0, [0], [(synth.token_major(k), synth.token_major(v))])
    q = th.zeros((11, 2, 128), dtype=th.float32, device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        c.prefill_attn(0, 0, q)
    assert e.value.code == kvq.KVQ_E_INVAL


@pytest.mark.parametrize("type_,hkv,n_q", [("kvarn4", 2, 64), ("q4_1", 1, 256)])
def test_prefill_chunk_at_64k_matches_oracle(type_, hkv, n_q):
    """Long context: a 64k-token cache (1024-token tail) and chunks of 64 and 256 queries, every
    query row against the oracle (several launches of 16 query tokens, each over the whole
    quantized prefix)."""
    th = H.torch()
    G, n, tail = 5, 65536, 1024
    rng = np.random.default_rng(n_q)
    k, v, _ = synth.kv_ar1(rng, hkv, n)
    c = H.make_cache(type_, hkv, n, tail)
    H.append(c, 0, [0], [(synth.token_major(k), synth.token_major(v))])
    q = rng.standard_normal((n_q, hkv * G, 128)).astype(np.float32)
    out = c.prefill_attn(0, 0, th.from_numpy(q).cuda())
    th.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    for h in range(hkv):
        ref = oracle.prefill_head(type_, type_, k[h], v[h], tail, q[:, h * G:(h + 1) * G])
        for i in range(n_q):
            H.check_decode(got[i, h * G:(h + 1) * G], ref[i], f"{type_} head {h} query {i}")
    assert c.status() == 0


QUANT_TYPES = [t for t in oracle.TYPES if t != "bf16"]


@pytest.mark.parametrize("type_", QUANT_TYPES)
def test_prefill_every_type(type_):
    """Every quantized type through the chunk kernel's tile rebuild (code widths 2 to 8, with and
    without a high plane, the three families): a 700-token cache with a 128-token tail and a
    150-query chunk (10 launches at GQA 4), whose early queries end inside the quantized prefix
    and whose quantized splits end in a partial tile."""
    th = H.torch()
    hkv, G, tail, n, n_q = 2, 4, 128, 700, 150
    rng = np.random.default_rng(7 + oracle.TYPES[type_])
    k, v, _ = synth.kv_ar1(rng, hkv, n)
    c = H.make_cache(type_, hkv, 1024, tail)
    H.append(c, 0, [0], [(synth.token_major(k), synth.token_major(v))])
    q = rng.standard_normal((n_q, hkv * G, 128)).astype(np.float32)
    out = c.prefill_attn(0, 0, th.from_numpy(q).cuda())
    th.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    for h in range(hkv):
        ref = oracle.prefill_head(type_, type_, k[h], v[h], tail, q[:, h * G:(h + 1) * G])
        for i in range(n_q):
            H.check_decode(got[i, h * G:(h + 1) * G], ref[i], f"{type_} head {h} query {i}")
    assert c.status() == 0


@pytest.mark.parametrize("type_", ["kvarn5", "q3_1", "bf16"])
def test_prefill_f16_tail(type_):
    """A cache with an F16 tail: the tail tiles are rebuilt from F16 ring rows; the reference is
    the oracle on the fp16-rounded inputs (the stream such a cache stores)."""
    th = H.torch()
    hkv, G, n, n_q = 2, 5, 600, 40
    tail = 0 if type_ == "bf16" else 100
    rng = np.random.default_rng(91)
    k, v, _ = synth.kv_ar1(rng, hkv, n)
    c = H.make_cache(type_, hkv, 1024, tail, tail_f16=1)
    H.append(c, 0, [0], [(synth.token_major(k), synth.token_major(v))])
    q = rng.standard_normal((n_q, hkv * G, 128)).astype(np.float32)
    out = c.prefill_attn(0, 0, th.from_numpy(q).cuda())
    th.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    for h in range(hkv):
        ref = oracle.prefill_head(type_, type_, oracle.f16_tail_rows(k[h]), oracle.f16_tail_rows(v[h]), tail,
                                  q[:, h * G:(h + 1) * G])
        for i in range(n_q):
            H.check_decode(got[i, h * G:(h + 1) * G], ref[i], f"{type_} head {h} query {i}")
    assert c.status() == 0
