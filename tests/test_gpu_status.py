"""The device status word: kernels that meet an inconsistent cache buffer record it and
carry on inside the buffer (no trap), and kvq_get_status reports it once.

The inconsistencies are made from the host, by writing into the caller-owned cache buffer
(a page-table entry outside the page pool, a merge ticket that is not zero), never by an
access outside any buffer: the kernels' own checks turn them into status bits."""
import numpy as np
import pytest

import gpu_helpers as H
from bit_kv_cache_17_b200 import kvq, synth

pytestmark = pytest.mark.gpu


def _cache_with_history():
    hkv, hq, n, tail = 2, 8, 700, 128
    rng = np.random.default_rng(31)
    k, v, _ = synth.kv_ar1(rng, hkv, n)
    c = H.make_cache("kvarn4", hkv, 1024, tail)
    H.append(c, 0, [0], [(synth.token_major(k), synth.token_major(v))])
    q = H.torch().from_numpy(synth.queries(rng, 1, 1, hq)[0]).cuda()
    return c, q, hq


def _poke(cache, off, value, dtype):
    t = H.torch()
    raw = np.array([value], dtype=dtype).view(np.uint8)
    cache.storage[off:off + raw.size] = t.from_numpy(raw.copy()).cuda()
    t.cuda.synchronize()


def test_page_table_entry_out_of_range_is_reported_and_contained():
    t = H.torch()
    c, q, hq = _cache_with_history()
    ref = c.decode(0, [0], q)
    assert c.status() == kvq.KVQ_OK
    off, nb = c.locate(2, 0, 0, 1, 0, 0)
    assert nb == 4
    orig = int(c.storage[off:off + 4].cpu().numpy().view(np.int32)[0])
    guard = c.storage[-4096:].clone()  # the end of the buffer (status word, tickets) stays put
    for bad in (0x7FFFFFFF, -5):
        _poke(c, off, bad, np.int32)
        out = c.decode(0, [0], q)
        assert c.status() == kvq.KVQ_E_DEVICE
        assert c.status() == kvq.KVQ_OK  # reading the word clears it
        assert t.isfinite(out).all()
        f = t.empty((300, 2, 128), dtype=t.float32, device="cuda")
        c.dequant(0, 0, 0, 200, 500, out=f)
        assert c.status() == kvq.KVQ_E_DEVICE
        _poke(c, off, orig, np.int32)
    out = c.decode(0, [0], q)
    assert c.status() == kvq.KVQ_OK
    H.check_decode(out.cpu().numpy(), ref.cpu().numpy().astype(np.float64), "restored page table")
    # only the status word (cleared again) and the merge tickets (reset by every merge) live there
    assert t.equal(c.storage[-4096:], guard)


def test_nonzero_merge_ticket_is_reported():
    t = H.torch()
    c, q, hq = _cache_with_history()
    ref = c.decode(0, [0], q)
    off, nb = c.locate(3, 0, 0, 0, 1, 0)  # decode entry 0, KV head 1
    assert nb == 4
    _poke(c, off, 1000, np.uint32)
    out = t.full_like(ref, float("nan"))
    c.decode(0, [0], q, out=out)
    assert c.status() == kvq.KVQ_E_DEVICE
    G = hq // 2
    # head 0 merged as usual; head 1 found no last block (its ticket never reached the count)
    H.check_decode(out[0, :G].cpu().numpy(), ref[0, :G].cpu().numpy().astype(np.float64), "head 0")
    assert t.isnan(out[0, G:]).all()
    _poke(c, off, 0, np.uint32)
    out = c.decode(0, [0], q)
    assert c.status() == kvq.KVQ_OK
    H.check_decode(out.cpu().numpy(), ref.cpu().numpy().astype(np.float64), "ticket reset")


def _gpus():
    try:
        return H.torch().cuda.device_count()
    except Exception:
        return 0


@pytest.mark.skipif(_gpus() < 2, reason="needs a second GPU to make current")
def test_calls_with_another_device_current_are_rejected_before_launch():
    t = H.torch()
    c, q, hq = _cache_with_history()
    out = t.zeros_like(q)
    n0 = kvq.kvq_launch_count()
    with t.cuda.device(1):
        for call in (lambda: c.decode(0, [0], q, out=out),
                     lambda: kvq.kvq_decode_attn_noalloc(c.handle, 0, [0], hq, q.data_ptr(), 0.0, out.data_ptr(), 0)):
            with pytest.raises(kvq.KVQError) as e:
                call()
            assert e.value.code == kvq.KVQ_E_INVAL
    assert kvq.kvq_launch_count() == n0
