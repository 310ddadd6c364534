"""GPU append path vs the oracle: packed codes and fp16 scales bit-exact, BF16 tail rows
bit-exact, whatever the append chunking (the cache state depends only on the tokens)."""
import numpy as np
import pytest

import gpu_helpers as H
from bit_kv_cache_17_b200 import synth

pytestmark = pytest.mark.gpu

QB = ["q2_0", "q3_0", "q4_0", "q5_0", "q6_0", "q8_0", "q4_1", "q2_1", "q3_1", "q5_1", "q6_1"]
KVARN = ["kvarn2", "kvarn3", "kvarn4", "kvarn5", "kvarn6", "kvarn8"]


def _data(hkv, n, seed, iid=False):
    rng = np.random.default_rng(seed)
    if iid:
        k, v = synth.kv_iid(rng, hkv, n)
    else:
        k, v, _ = synth.kv_ar1(rng, hkv, n)
    return k, v  # [hkv, n, 128]


def _check_all(cache, type_, layer, seq, k, v, tail):
    buf = H.storage_bytes(cache)
    for h in range(k.shape[0]):
        H.compare_stream(cache, buf, type_, layer, seq, h, 0, k[h], tail)
        H.compare_stream(cache, buf, type_, layer, seq, h, 1, v[h], tail)


def test_config0_kvarn4_bitexact():
    cfg = synth.config0()
    k, v = cfg["k"], cfg["v"]
    c = H.make_cache("kvarn4", cfg["hkv"], cfg["n"], cfg["tail"])
    H.append(c, 0, [0], [(synth.token_major(k), synth.token_major(v))])
    assert c.seq_len(0, 0) == 2048
    _check_all(c, "kvarn4", 0, 0, k, v, cfg["tail"])
    assert c.status() == 0


@pytest.mark.parametrize("t", QB + KVARN)
@pytest.mark.parametrize("tail", [0, 300])
def test_every_type_bitexact(t, tail):
    k, v = _data(2, 1100, 11)
    c = H.make_cache(t, 2, 1200, tail)
    H.append(c, 0, [0], [(synth.token_major(k[:, :700]), synth.token_major(v[:, :700]))])
    H.append(c, 0, [0], [(synth.token_major(k[:, 700:]), synth.token_major(v[:, 700:]))])
    _check_all(c, t, 0, 0, k, v, tail)


@pytest.mark.parametrize("t", ["kvarn4", "q3_1", "kvarn3"])
def test_chunking_invariance_multi_sequence(t):
    """Sequences appended in different chunkings (single tokens, ragged chunks, one call)
    within shared batched calls end in the oracle's from-scratch state."""
    hkv, tail = 2, 100
    data = [_data(hkv, n, 20 + i) for i, n in enumerate((900, 613, 300))]
    chunkings = [[1] * 40 + [860], [255, 1, 256, 100, 1], [300]]
    c = H.make_cache(t, hkv, 1024, tail, n_seqs=3)
    pos = [0, 0, 0]
    plans = [list(ch) for ch in chunkings]
    while any(plans):
        ids, rows = [], []
        for s in range(3):
            if plans[s]:
                m = plans[s].pop(0)
                k, v = data[s]
                ids.append(s)
                rows.append((synth.token_major(k[:, pos[s]:pos[s] + m]), synth.token_major(v[:, pos[s]:pos[s] + m])))
                pos[s] += m
        # reverse the order of the sequences in the call to exercise the input offsets
        H.append(c, 0, ids[::-1], rows[::-1])
    for s in range(3):
        k, v = data[s]
        n = pos[s]
        assert c.seq_len(0, s) == n
        buf = H.storage_bytes(c)
        for h in range(hkv):
            H.compare_stream(c, buf, t, 0, s, h, 0, k[h, :n], tail)
            H.compare_stream(c, buf, t, 0, s, h, 1, v[h, :n], tail)


def test_single_token_steps_across_group_boundaries():
    """The decode-step pattern: one token per call while the oldest tail token spills into
    a growing kvarn group (a new group every 256 steps)."""
    hkv, tail = 1, 64
    k, v = _data(hkv, 900, 31)
    c = H.make_cache("kvarn2", hkv, 1024, tail)
    H.append(c, 0, [0], [(synth.token_major(k[:, :250]), synth.token_major(v[:, :250]))])
    for p in range(250, 900):
        H.append(c, 0, [0], [(synth.token_major(k[:, p:p + 1]), synth.token_major(v[:, p:p + 1]))])
        if p in (250 + tail, 256 + tail, 511 + tail, 512 + tail, 899):
            _check_all(c, "kvarn2", 0, 0, k[:, :p + 1], v[:, :p + 1], tail)


def test_short_sequences_stay_in_the_tail_and_layers_are_separate():
    hkv, tail = 2, 512
    k, v = _data(hkv, 600, 41)
    c = H.make_cache("kvarn4", hkv, 700, tail, n_layers=2)
    H.append(c, 1, [0], [(synth.token_major(k[:, :500]), synth.token_major(v[:, :500]))])
    assert c.seq_len(0, 0) == 0 and c.seq_len(1, 0) == 500
    _check_all(c, "kvarn4", 1, 0, k[:, :500], v[:, :500], tail)
    H.append(c, 1, [0], [(synth.token_major(k[:, 500:]), synth.token_major(v[:, 500:]))])
    _check_all(c, "kvarn4", 1, 0, k, v, tail)


def test_capacity_and_argument_errors():
    from bit_kv_cache_17_b200 import kvq

    k, v = _data(1, 40, 51)
    c = H.make_cache("q4_0", 1, 32, 8)
    with pytest.raises(kvq.KVQError) as e:
        H.append(c, 0, [0], [(synth.token_major(k), synth.token_major(v))])
    assert e.value.code == kvq.KVQ_E_CAPACITY
    assert c.seq_len(0, 0) == 0
    with pytest.raises(kvq.KVQError) as e:
        H.append(c, 0, [0, 0], [(synth.token_major(k[:, :2]), synth.token_major(v[:, :2]))] * 2)
    assert e.value.code == kvq.KVQ_E_INVAL
    with pytest.raises(kvq.KVQError) as e:
        H.append(c, 1, [0], [(synth.token_major(k[:, :2]), synth.token_major(v[:, :2]))])
    assert e.value.code == kvq.KVQ_E_INVAL
    assert c.status() == 0
