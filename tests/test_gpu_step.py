"""kvq_append_decode (append, then decode of the same sequences, the decode overlapping the
append) against the CPU oracle: every packed byte and ring row of the sampled streams equals
the oracle's state of the full history, and the decode output agrees with the oracle's
decode of that history (relative L2 <= 1e-3, max abs <= 2e-3 x RMS).

Cases: one-token kvarn steps (the spill kernel writes the ring rows itself) that cross a
256-token group boundary; a multi-token kvarn append (separate ring write); a q4_0 cache
(separate ring write, qb spill); sequences appended with zero tokens next to appended ones;
and the decode workload at 64k context."""
import numpy as np
import pytest

import gpu_helpers as H
from bit_kv_cache_17_b200 import synth

pytestmark = pytest.mark.gpu


def _rows(x, a, b):
    return synth.token_major(x[:, a:b])


def _check(c, type_, data, lens, tail, seq_ids, q, out):
    buf = H.storage_bytes(c)
    for row, s in enumerate(seq_ids):
        k, v = data[s]
        n = lens[s]
        for h in range(k.shape[0]):
            H.compare_stream(c, buf, type_, 0, s, h, 0, k[h, :n], tail)
            H.compare_stream(c, buf, type_, 0, s, h, 1, v[h, :n], tail)
        ref = H.oracle_decode(type_, k[:, :n], v[:, :n], tail, q[row])
        H.check_decode(out[row], ref, f"{type_} seq {s} n {n}")


@pytest.mark.parametrize("type_,steps", [("kvarn4", [1, 1, 1, 1, 1]), ("kvarn2", [1, 37, 1]), ("q4_0", [1, 1, 5])])
def test_append_decode_matches_oracle(type_, steps):
    th = H.torch()
    hkv, hq, tail = 2, 10, 200
    rng = np.random.default_rng(31)
    total = 1800
    data = [synth.kv_ar1(rng, hkv, total)[:2] for _ in range(2)]
    # sequence 0 ends its prefill 2 tokens before a group boundary of the quantized prefix,
    # so that one-token steps spill into a fresh group
    lens = [200 + 3 * 256 - 2, 900]
    c = H.make_cache(type_, hkv, 2048, tail, n_seqs=2)
    H.append(c, 0, [0, 1], [(_rows(data[s][0], 0, lens[s]), _rows(data[s][1], 0, lens[s])) for s in range(2)])
    for st, n_new in enumerate(steps):
        # sequence 1 takes no new token on odd steps
        new = [n_new, 0 if st % 2 else n_new]
        k = np.concatenate([_rows(data[s][0], lens[s], lens[s] + new[s]) for s in range(2)])
        v = np.concatenate([_rows(data[s][1], lens[s], lens[s] + new[s]) for s in range(2)])
        q = synth.queries(rng, 1, 2, hq)[0]
        out = c.append_decode(0, [1, 0], [new[1], new[0]],
                              H.to_dev_bf16(np.concatenate([k[new[0]:], k[:new[0]]])),
                              H.to_dev_bf16(np.concatenate([v[new[0]:], v[:new[0]]])),
                              th.from_numpy(q).cuda())
        th.cuda.synchronize()
        for s in range(2):
            lens[s] += new[s]
        _check(c, type_, data, lens, tail, [1, 0], q, out.cpu().numpy().astype(np.float64))
    assert c.status() == 0


def test_append_decode_64k():
    th = H.torch()
    cfg = synth.config2()
    n, hkv, hq, tail = cfg["n"], cfg["hkv"], cfg["hq"], cfg["tail"]
    c = H.make_cache("kvarn4", hkv, n, tail)
    kt, vt = H.to_dev_bf16(synth.token_major(cfg["k"])), H.to_dev_bf16(synth.token_major(cfg["v"]))
    P = n - 3
    c.append(0, [0], [P], kt[:P], vt[:P])
    for i in range(3):
        q = cfg["q"][i, 0]
        out = c.append_decode(0, [0], [1], kt[P + i:P + i + 1], vt[P + i:P + i + 1], th.from_numpy(q).cuda()[None])
    th.cuda.synchronize()
    got = out.cpu().numpy()[0].astype(np.float64)
    buf = H.storage_bytes(c)
    G = hq // hkv
    import oracle

    for h in (0, 7):
        H.compare_stream(c, buf, "kvarn4", 0, 0, h, 0, cfg["k"][h], tail)
        H.compare_stream(c, buf, "kvarn4", 0, 0, h, 1, cfg["v"][h], tail)
        ref = oracle.decode_head("kvarn4", "kvarn4", cfg["k"][h], cfg["v"][h], tail, q[h * G:(h + 1) * G])
        H.check_decode(got[h * G:(h + 1) * G], ref, f"64k head {h}")
    assert c.status() == 0


@pytest.mark.parametrize("type_", ["bf16", "q8_0"])
def test_append_decode_short_context_and_bf16(type_):
    """A BF16 cache (every row in the ring: the decode follows the ring-write kernel) and a
    q8_0 cache whose first steps do not spill (context below the tail)."""
    th = H.torch()
    hkv, hq, tail = 2, 8, 64
    rng = np.random.default_rng(41)
    k, v, _ = synth.kv_ar1(rng, hkv, 120)
    c = H.make_cache(type_, hkv, 256, tail if type_ != "bf16" else 0)
    n = 40
    c.append(0, [0], [n], H.to_dev_bf16(_rows(k, 0, n)), H.to_dev_bf16(_rows(v, 0, n)))
    for step in range(4):
        m = 1 if step < 3 else 30  # the last step crosses the tail and spills
        q = synth.queries(rng, 1, 1, hq)[0]
        out = c.append_decode(0, [0], [m], H.to_dev_bf16(_rows(k, n, n + m)), H.to_dev_bf16(_rows(v, n, n + m)),
                              th.from_numpy(q).cuda())
        th.cuda.synchronize()
        n += m
        _check(c, type_, [(k, v)], [n], tail if type_ != "bf16" else 0, [0], q, out.cpu().numpy().astype(np.float64))
    assert c.status() == 0


def test_append_decode_more_sequences_than_one_launch():
    """70 sequences: the append and the decode each take two launches (64 sequences per
    launch), so the decode is not overlapped; every output still matches the oracle."""
    th = H.torch()
    hkv, hq, tail, S = 1, 2, 32, 70
    rng = np.random.default_rng(43)
    lens = [int(x) for x in rng.integers(1, 200, S)]
    data = [synth.kv_ar1(rng, hkv, lens[s] + 1)[:2] for s in range(S)]
    c = H.make_cache("kvarn3", hkv, 256, tail, n_seqs=S)
    H.append(c, 0, list(range(S)), [(_rows(data[s][0], 0, lens[s]), _rows(data[s][1], 0, lens[s])) for s in range(S)])
    q = synth.queries(rng, 1, S, hq)[0]
    ids = list(range(S))[::-1]
    k = np.concatenate([_rows(data[s][0], lens[s], lens[s] + 1) for s in ids])
    v = np.concatenate([_rows(data[s][1], lens[s], lens[s] + 1) for s in ids])
    out = c.append_decode(0, ids, [1] * S, H.to_dev_bf16(k), H.to_dev_bf16(v), th.from_numpy(q).cuda())
    th.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    for row, s in enumerate(ids):
        kk, vv = data[s]
        n = lens[s] + 1
        ref = H.oracle_decode("kvarn3", kk[:, :n], vv[:, :n], tail, q[row])
        H.check_decode(got[row], ref, f"seq {s}")
    assert c.status() == 0
