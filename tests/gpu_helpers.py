"""Helpers shared by the GPU parity tests: build caches through the C ABI, read their
bytes back, and compare them with the oracle's state of the same streams."""
import numpy as np

import oracle

D = 128

TOL_REL_L2 = 1e-3      # decode: relative L2 error against the fp64 oracle
TOL_MAX_ABS = 2e-3     # decode: max abs error, times the RMS of the oracle output


def torch():
    import torch as t

    return t


def make_cache(type_k, hkv, max_ctx, tail, n_seqs=1, n_layers=1, type_v=None, iters=8, tail_f16=0):
    from bit_kv_cache_17_b200.kvq import KVCache

    return KVCache(n_layers=n_layers, n_seqs=n_seqs, n_kv_heads=hkv, max_ctx=max_ctx, type_k=type_k,
                   type_v=type_v or type_k, tail=tail, sinkhorn_iters=iters, tail_f16=tail_f16)


def to_dev_bf16(tok_major_bits):
    t = torch()
    a = np.ascontiguousarray(tok_major_bits.astype(np.uint16))
    return t.from_numpy(a.view(np.int16)).view(t.bfloat16).cuda()


def append(cache, layer, seq_ids, rows_per_seq):
    """rows_per_seq: list of (k [n, hkv, 128] bits, v [n, hkv, 128] bits) in seq_ids order"""
    ks = np.concatenate([r[0] for r in rows_per_seq], axis=0)
    vs = np.concatenate([r[1] for r in rows_per_seq], axis=0)
    cache.append(layer, seq_ids, [r[0].shape[0] for r in rows_per_seq], to_dev_bf16(ks), to_dev_bf16(vs))


def storage_bytes(cache):
    torch().cuda.synchronize()
    return cache.storage.cpu().numpy()


def compare_stream(cache, buf, type_, layer, seq, head, which, hist, tail, ring_bits=None):
    """hist: [n, 128] BF16 bits of one stream.  Quantized sub-pages must equal the oracle's
    images on every byte of a valid token; tail rows must equal the input bits (or ring_bits,
    the stored 16-bit rows, for an F16 tail)."""
    n = hist.shape[0]
    st = oracle.stream_state(type_, hist, tail)
    Q = st["Q"]
    mism = 0
    if oracle.family(type_) != 0:
        for page in range((Q + 255) // 256):
            img, mask = oracle.pack_subpage(type_, which, st, page)
            off, nb = cache.locate(0, layer, seq, page, head, which)
            got = buf[off:off + nb]
            m = mask.astype(bool)
            bad = np.nonzero(got[m] != img[m])[0]
            mism += len(bad)
            assert len(bad) == 0, (type_, seq, head, which, page, len(bad))
    keep0 = Q if oracle.family(type_) != 3 else (Q // 256) * 256
    for p in range(keep0, n):
        off, nb = cache.locate(1, layer, seq, 0, head, which, p)
        got = buf[off:off + nb].view(np.uint16)
        want = hist[p] if ring_bits is None else ring_bits[p]
        assert np.array_equal(got, want), (type_, seq, head, which, p)
    return Q


def check_decode(out_gpu, out_ref, what=""):
    out_gpu = np.asarray(out_gpu, dtype=np.float64)
    rel = np.linalg.norm(out_gpu - out_ref) / max(np.linalg.norm(out_ref), 1e-300)
    rms = np.sqrt(np.mean(out_ref**2))
    mx = np.max(np.abs(out_gpu - out_ref)) / max(rms, 1e-300)
    assert rel <= TOL_REL_L2 and mx <= TOL_MAX_ABS, (what, rel, mx)
    return rel, mx


def oracle_decode(type_, hists_k, hists_v, tail, q, scale=None):
    """q: [Hq, 128] fp32 for one sequence; hists: per KV head [n, 128] bits."""
    hkv = len(hists_k)
    G = q.shape[0] // hkv
    out = np.zeros((q.shape[0], D))
    for h in range(hkv):
        out[h * G:(h + 1) * G] = oracle.decode_head(type_, type_, hists_k[h], hists_v[h], tail,
                                                    q[h * G:(h + 1) * G], scale)
    return out
