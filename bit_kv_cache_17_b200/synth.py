"""Seeded synthetic inputs for the KV-cache workloads (numpy only).

This module holds no step of the method: it draws K/V head vectors and queries and
rounds K/V to BF16 (the cache's input format).  Both the CUDA path and the CPU oracle
consume what it returns; neither is imported here.

Recipe (one generator per workload, numpy PCG64 `default_rng(seed)`, float64 draws):
  * i.i.d. data: K, V ~ N(0, 1) per (KV head, token, channel);
  * AR(1) data: per (KV head, channel) along tokens, x_0 = e_0 / sqrt(1 - rho^2),
    x_t = rho x_{t-1} + e_t, rho = 0.9, e ~ N(0, 1);
  * draw order: K innovations [Hkv, N, 128], V innovations, then (AR(1) data) 4 outlier
    channels per KV head (`rng.choice(128, 4, replace=False)`, head by head), then the
    queries `standard_normal((steps, batch, Hq, 128))`;
  * K outlier channels are multiplied (x16 for i.i.d. data on channels 7 and 63, x20 for
    AR(1) data on the drawn channels) before K and V are cast to fp32 and rounded to BF16
    (round to nearest, ties to even); queries stay fp32.
"""
import numpy as np
from scipy.signal import lfilter

D = 128


def bf16_bits(x):
    """fp32 -> BF16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + (0x7FFF + ((u >> 16) & 1))) >> 16).astype(np.uint16)


def bf16_to_f32(h):
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _ar1(eps, rho):
    eps[:, 0, :] /= np.sqrt(1.0 - rho * rho)
    return lfilter([1.0], [1.0, -rho], eps, axis=1)


def kv_iid(rng, hkv, n, outlier_channels=(7, 63), factor=16.0):
    k = rng.standard_normal((hkv, n, D))
    v = rng.standard_normal((hkv, n, D))
    for ch in outlier_channels:
        k[:, :, ch] *= factor
    return bf16_bits(k.astype(np.float32)), bf16_bits(v.astype(np.float32))


def kv_ar1(rng, hkv, n, rho=0.9, n_outliers=4, factor=20.0):
    k = _ar1(rng.standard_normal((hkv, n, D)), rho)
    v = _ar1(rng.standard_normal((hkv, n, D)), rho)
    outl = [rng.choice(D, n_outliers, replace=False) for _ in range(hkv)]
    for h in range(hkv):
        k[h][:, outl[h]] *= factor
    kb = bf16_bits(k.astype(np.float32))
    del k
    vb = bf16_bits(v.astype(np.float32))
    return kb, vb, outl


def queries(rng, steps, batch, hq):
    return rng.standard_normal((steps, batch, hq, D)).astype(np.float32)


# ---------------------------------------------------------------------------------------
# workloads.  K/V arrays are [Hkv, N, 128] BF16 bits (uint16); queries [steps, B, Hq, 128]

def config0():
    """One layer, batch 1, 4 KV heads, 16 query heads, context 2048 (1792 kvarn4 + 256 BF16
    tail), i.i.d. N(0,1) K/V, K channels 7 and 63 x16, one decode step, seed 0."""
    rng = np.random.default_rng(0)
    hkv, hq, n = 4, 16, 2048
    k, v = kv_iid(rng, hkv, n)
    q = queries(rng, 1, 1, hq)
    return dict(name="cfg0", hkv=hkv, hq=hq, n=n, tail=256, types=["kvarn4"], k=k, v=v, q=q, seed=0)


def config1(n=16384, hkv=8, hq=32):
    """Plain block formats: 8 KV heads, 32 query heads, context 16384, tails 0/1024/2048,
    AR(1) K/V with 4 outlier channels x20 in K, seed 1."""
    rng = np.random.default_rng(1)
    k, v, _ = kv_ar1(rng, hkv, n)
    q = queries(rng, 1, 1, hq)
    return dict(name="cfg1", hkv=hkv, hq=hq, n=n, tails=[0, 1024, 2048],
                types=["q2_0", "q3_0", "q4_0", "q5_0", "q6_0", "q8_0", "q4_1"], k=k, v=v, q=q, seed=1)


def config2(n=65536, steps=128, hkv=8, hq=40):
    """kvarn2..kvarn8 at context 65536 with a 1024-token tail, 8 KV heads, 40 query heads;
    128 decode steps each appending one token (the cache holds n - steps tokens before the
    first step); AR(1) data as config 1, seed 2."""
    rng = np.random.default_rng(2)
    k, v, _ = kv_ar1(rng, hkv, n)
    q = queries(rng, steps, 1, hq)
    return dict(name="cfg2", hkv=hkv, hq=hq, n=n, steps=steps, tail=1024,
                types=["kvarn2", "kvarn3", "kvarn4", "kvarn5", "kvarn6", "kvarn8"], k=k, v=v, q=q, seed=2)


def config3_lengths():
    return np.random.default_rng(3).integers(4096, 32768, 16, endpoint=True)


def config3(n_seqs=16, prefill=4096, steps=64, hkv=8, hq=32, lengths=None):
    """Batched serving: 16 sequences with lengths L_i ~ U[4096, 32768] (seeded), kvarn4
    with a 1024-token tail; each sequence is built to L_i, then appends `prefill` tokens
    in one call, then `steps` batched decode steps (one token each); AR(1) data, seed 3.
    Per sequence K/V hold L_i + prefill + steps rows."""
    rng = np.random.default_rng(3)
    L = rng.integers(4096, 32768, 16, endpoint=True)[:n_seqs]
    if lengths is not None:
        L = np.asarray(lengths)
    ks, vs = [], []
    for i in range(len(L)):
        k, v, _ = kv_ar1(rng, hkv, int(L[i]) + prefill + steps)
        ks.append(k)
        vs.append(v)
    q = queries(rng, steps, len(L), hq)
    return dict(name="cfg3", hkv=hkv, hq=hq, lengths=[int(x) for x in L], prefill=prefill, steps=steps,
                tail=1024, types=["kvarn4"], k=ks, v=vs, q=q, seed=3)


def config4_layer(layer, n=240000, hkv=8, hq=64):
    """Page-1 shape, one layer: 8 KV heads, 64 query heads, context 240000, AR(1) data as
    config 1 seeded by the layer index; kvarn2 / q4_0 with a 1024-token tail, and BF16."""
    rng = np.random.default_rng(layer)
    k, v, _ = kv_ar1(rng, hkv, n)
    q = queries(rng, 1, 1, hq)
    return dict(name="cfg4", layer=layer, hkv=hkv, hq=hq, n=n, tail=1024, types=["kvarn2", "q4_0", "bf16"],
                k=k, v=v, q=q, seed=layer)


def token_major(kv):
    """[Hkv, N, 128] -> [N, Hkv, 128] (the append input layout), contiguous."""
    return np.ascontiguousarray(np.transpose(kv, (1, 0, 2)))
