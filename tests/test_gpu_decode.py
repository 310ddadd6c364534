"""GPU decode attention vs the fp64 oracle on the same seeded inputs: relative L2 error
<= 1e-3 and max abs error <= 2e-3 x output RMS (fp32 accumulation on the GPU)."""
import numpy as np
import pytest

import gpu_helpers as H
from bit_kv_cache_17_b200 import synth

pytestmark = pytest.mark.gpu

TYPES = ["bf16", "q2_0", "q3_0", "q4_0", "q5_0", "q6_0", "q8_0", "q4_1", "q2_1", "q3_1", "q5_1", "q6_1",
         "kvarn2", "kvarn3", "kvarn4", "kvarn5", "kvarn6", "kvarn8"]


def _decode(cache, layer, seq_ids, q):
    t = H.torch()
    qd = t.from_numpy(np.ascontiguousarray(q, dtype=np.float32)).cuda()
    out = cache.decode(layer, seq_ids, qd)
    t.cuda.synchronize()
    return out.cpu().numpy()


def test_config0():
    cfg = synth.config0()
    k, v, q = cfg["k"], cfg["v"], cfg["q"][0]
    c = H.make_cache("kvarn4", cfg["hkv"], cfg["n"], cfg["tail"])
    H.append(c, 0, [0], [(synth.token_major(k), synth.token_major(v))])
    out = _decode(c, 0, [0], q)[0]
    ref = H.oracle_decode("kvarn4", k, v, cfg["tail"], q[0])
    H.check_decode(out, ref, "cfg0")
    assert c.status() == 0


@pytest.mark.parametrize("t", TYPES)
def test_every_type(t):
    hkv, hq, n, tail = 2, 10, 1500, 200
    rng = np.random.default_rng(7)
    k, v, _ = synth.kv_ar1(rng, hkv, n)
    q = synth.queries(rng, 1, 1, hq)[0]
    c = H.make_cache(t, hkv, 2048, tail)
    H.append(c, 0, [0], [(synth.token_major(k), synth.token_major(v))])
    out = _decode(c, 0, [0], q)[0]
    ref = H.oracle_decode(t, k, v, tail if t != "bf16" else 0, q[0])
    H.check_decode(out, ref, t)


@pytest.mark.parametrize("G", [1, 3, 8])
def test_gqa_and_batched_ragged_sequences(G):
    """Several sequences of ragged lengths (empty, shorter than the tail, a partial group,
    several pages) decoded in one call; query rows follow the order of the call."""
    hkv, tail = 2, 96
    lens = [0, 50, 96, 97, 300, 777]
    rng = np.random.default_rng(100 + G)
    data = [synth.kv_ar1(rng, hkv, max(n, 1))[:2] for n in lens]
    c = H.make_cache("kvarn3", hkv, 1024, tail, n_seqs=len(lens))
    ids = [s for s in range(len(lens)) if lens[s] > 0]
    H.append(c, 0, ids, [(synth.token_major(data[s][0][:, :lens[s]]), synth.token_major(data[s][1][:, :lens[s]]))
                         for s in ids])
    order = [5, 0, 3, 1, 4, 2]
    q = synth.queries(rng, 1, len(order), hkv * G)[0]
    out = _decode(c, 0, order, q)
    for row, s in enumerate(order):
        if lens[s] == 0:
            assert not out[row].any()
            continue
        k, v = data[s]
        ref = H.oracle_decode("kvarn3", k[:, :lens[s]], v[:, :lens[s]], tail, q[row])
        H.check_decode(out[row], ref, f"seq {s}")


def test_softmax_scale_and_workspace_errors():
    from bit_kv_cache_17_b200 import kvq

    hkv, n = 1, 400
    rng = np.random.default_rng(9)
    k, v, _ = synth.kv_ar1(rng, hkv, n)
    q = synth.queries(rng, 1, 1, 4)[0]
    c = H.make_cache("q8_0", hkv, 512, 64)
    H.append(c, 0, [0], [(synth.token_major(k), synth.token_major(v))])
    t = H.torch()
    qd = t.from_numpy(q).cuda()
    out = c.decode(0, [0], qd, softmax_scale=0.05)
    ref = H.oracle_decode("q8_0", k, v, 64, q[0], scale=0.05)
    H.check_decode(out.cpu().numpy()[0], ref, "scale")
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_decode_attn(c.handle, 0, [0], 4, qd.data_ptr(), 0.0, out.data_ptr(), c._ws.data_ptr(), 16, 0)
    assert e.value.code == kvq.KVQ_E_SIZE
    q9 = t.zeros((1, 9, 128), device="cuda")
    with pytest.raises(kvq.KVQError) as e:
        c.decode(0, [0], q9)
    assert e.value.code == kvq.KVQ_E_UNSUPPORTED
