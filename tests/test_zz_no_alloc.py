"""kvq_decode_attn_noalloc: decode attention for callers that cannot allocate device
memory (a plugin whose host runtime owns all device memory, a serving loop that must not
allocate once running).  It keeps its split-K partials in a fixed library-owned device
array instead of a caller workspace.  Checked through the C ABI against kvq_decode_attn
on two calls in a row; this file is collected last so that a failure here comes after
every other test has run."""
import numpy as np
import pytest

import gpu_helpers as H
from bit_kv_cache_17_b200 import kvq, synth

pytestmark = pytest.mark.gpu


def test_noalloc_decode_matches_workspace_decode_twice():
    t = H.torch()
    hkv, hq, n, tail = 4, 20, 3000, 512
    rng = np.random.default_rng(77)
    k, v, _ = synth.kv_ar1(rng, hkv, n + 2)
    c = H.make_cache("kvarn4", hkv, 4096, tail, n_seqs=2)
    H.append(c, 0, [0, 1], [(synth.token_major(k[:, :n]), synth.token_major(v[:, :n])),
                            (synth.token_major(k[:, :700]), synth.token_major(v[:, :700]))])
    for call in range(2):
        q = t.from_numpy(synth.queries(rng, 1, 2, hq)[0]).cuda()
        ref = c.decode(0, [1, 0], q)
        got = t.full_like(q, float("nan"))
        kvq.kvq_decode_attn_noalloc(c.handle, 0, [1, 0], hq, q.data_ptr(), 0.0, got.data_ptr(),
                                    t.cuda.current_stream().cuda_stream)
        t.cuda.synchronize()
        for row in range(2):
            H.check_decode(got[row].cpu().numpy(), ref[row].cpu().numpy().astype(np.float64), f"call {call}")
        # one more token per sequence between the two calls
        a, b = n + call, 700 + call
        H.append(c, 0, [0, 1], [(synth.token_major(k[:, a:a + 1]), synth.token_major(v[:, a:a + 1])),
                                (synth.token_major(k[:, b:b + 1]), synth.token_major(v[:, b:b + 1]))])
    assert c.status() == 0


def test_noalloc_rejects_work_beyond_its_array():
    t = H.torch()
    c = H.make_cache("q4_0", 8, 512, 64, n_seqs=16)
    q = t.zeros((16, 64, 128), dtype=t.float32, device="cuda")
    out = t.zeros_like(q)
    need = kvq.kvq_workspace_bytes(c.handle, 16, 64)
    assert need > (4 << 20)
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_decode_attn_noalloc(c.handle, 0, list(range(16)), 64, q.data_ptr(), 0.0, out.data_ptr(), 0)
    assert e.value.code == kvq.KVQ_E_SIZE


def test_noalloc_mixed_types_match_workspace_decode_twice():
    """K and V of different types also keep the Q.K scores of the quantized prefix in the
    array (two kernels over one split plan)."""
    t = H.torch()
    hkv, hq, n, tail = 2, 10, 1500, 256
    rng = np.random.default_rng(78)
    k, v, _ = synth.kv_ar1(rng, hkv, n + 2)
    c = H.make_cache("kvarn4", hkv, 2048, tail, type_v="q4_0")
    H.append(c, 0, [0], [(synth.token_major(k[:, :n]), synth.token_major(v[:, :n]))])
    for call in range(2):
        q = t.from_numpy(synth.queries(rng, 1, 1, hq)[0]).cuda()
        ref = c.decode(0, [0], q)
        got = t.full_like(q, float("nan"))
        kvq.kvq_decode_attn_noalloc(c.handle, 0, [0], hq, q.data_ptr(), 0.0, got.data_ptr(),
                                    t.cuda.current_stream().cuda_stream)
        t.cuda.synchronize()
        H.check_decode(got[0].cpu().numpy(), ref[0].cpu().numpy().astype(np.float64), f"mixed call {call}")
        a = n + call
        H.append(c, 0, [0], [(synth.token_major(k[:, a:a + 1]), synth.token_major(v[:, a:a + 1]))])
    assert c.status() == 0


def test_noalloc_mixed_type_limit_is_the_documented_one():
    """8 KV heads, GQA 5, one sequence of a mixed K/V cache: max_ctx 17 760 fits the array,
    17 761 does not (the score rows are rounded up to 32 tokens)."""
    t = H.torch()
    q = t.zeros((1, 40, 128), dtype=t.float32, device="cuda")
    out = t.zeros_like(q)
    for max_ctx, fits in ((17760, True), (17761, False)):
        c = H.make_cache("kvarn4", 8, max_ctx, 64, type_v="q4_0")
        need = kvq.kvq_workspace_bytes(c.handle, 1, 40)
        assert (need <= (4 << 20)) == fits, (max_ctx, need)
        if fits:
            kvq.kvq_decode_attn_noalloc(c.handle, 0, [0], 40, q.data_ptr(), 0.0, out.data_ptr(), 0)
        else:
            with pytest.raises(kvq.KVQError) as e:
                kvq.kvq_decode_attn_noalloc(c.handle, 0, [0], 40, q.data_ptr(), 0.0, out.data_ptr(), 0)
            assert e.value.code == kvq.KVQ_E_SIZE
        t.cuda.synchronize()
        del c
