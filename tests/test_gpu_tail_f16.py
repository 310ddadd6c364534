"""A cache with an F16 tail ("KV Cache Precision Tail": the newest tokens stay 16-bit, BF16
or F16) against the CPU oracle.  The tail stores fp16(x) of each BF16 input and tokens are
quantized from that value; since every fp16 rounding of a BF16 value is a BF16 value, the
oracle's BF16-tail stream of the rounded rows is the reference.

The data puts three channels of every head in the fp16 subnormal range (x 2^-20), where the
rounding changes the values, so every conversion path shows: ring writes (separate and fused
into the spill), quantization from the input and from the ring, the decode's f16 tensor-core
tail path, and the dequant read-back."""
import numpy as np
import pytest

import gpu_helpers as H
import oracle
from bit_kv_cache_17_b200 import synth

pytestmark = pytest.mark.gpu

TINY = (3, 50, 97)


def _data(rng, hkv, n):
    k, v, _ = synth.kv_ar1(rng, hkv, n)
    out = []
    for x in (k, v):
        f = oracle.bf16_to_f32(x).copy()
        f[:, :, TINY] *= 2.0**-20
        out.append(oracle.f32_to_bf16(f))
    return out


def _rows(x, a, b):
    return synth.token_major(x[:, a:b])


def _check_streams(c, type_, k, v, n, tail):
    buf = H.storage_bytes(c)
    for h in range(k.shape[0]):
        for which, x in ((0, k), (1, v)):
            H.compare_stream(c, buf, type_, 0, 0, h, which, oracle.f16_tail_rows(x[h, :n]), tail,
                             ring_bits=oracle.f16_tail_bits(x[h, :n]))


def _ref(type_, k, v, n, tail, q, hkv):
    G = q.shape[0] // hkv
    out = np.zeros((q.shape[0], 128))
    for h in range(hkv):
        out[h * G:(h + 1) * G] = oracle.decode_head(type_, type_, oracle.f16_tail_rows(k[h, :n]),
                                                    oracle.f16_tail_rows(v[h, :n]), tail, q[h * G:(h + 1) * G])
    return out


@pytest.mark.parametrize("type_", ["kvarn4", "q4_0", "q4_1", "bf16"])
def test_f16_tail_streams_and_decode(type_):
    th = H.torch()
    hkv, hq, tail = 2, 10, 100
    tl = tail if type_ != "bf16" else 0
    n = 100 + 2 * 256 + 37
    rng = np.random.default_rng(61)
    k, v = _data(rng, hkv, n)
    c = H.make_cache(type_, hkv, 1024, tl, tail_f16=1)
    H.append(c, 0, [0], [(_rows(k, 0, n), _rows(v, 0, n))])
    q = synth.queries(rng, 1, 1, hq)[0]
    out = c.decode(0, [0], th.from_numpy(q).cuda())
    th.cuda.synchronize()
    _check_streams(c, type_, k, v, n, tl)
    H.check_decode(out.cpu().numpy()[0].astype(np.float64), _ref(type_, k, v, n, tl, q[0], hkv), type_)
    # the tail reads back as the stored fp16 values
    a = n - min(n, tl) if type_ != "bf16" else 0
    got = c.dequant(0, 0, 1, a, n).cpu().numpy()
    want = oracle.f16_to_f32(oracle.f16_tail_bits(np.transpose(v[:, a:n], (1, 0, 2))))
    assert np.array_equal(got, want)
    assert c.status() == 0


def test_f16_tail_one_token_steps():
    """kvarn3, one-token steps across a group boundary: the spill re-quantizes the open group
    from F16 ring rows and writes the new row itself."""
    th = H.torch()
    hkv, hq, tail = 2, 8, 64
    rng = np.random.default_rng(67)
    n = 64 + 256 - 3
    k, v = _data(rng, hkv, n + 6)
    c = H.make_cache("kvarn3", hkv, 1024, tail, tail_f16=1)
    H.append(c, 0, [0], [(_rows(k, 0, n), _rows(v, 0, n))])
    for step in range(6):
        q = synth.queries(rng, 1, 1, hq)[0]
        out = c.append_decode(0, [0], [1], H.to_dev_bf16(_rows(k, n, n + 1)), H.to_dev_bf16(_rows(v, n, n + 1)),
                              th.from_numpy(q).cuda())
        th.cuda.synchronize()
        n += 1
        _check_streams(c, "kvarn3", k, v, n, tail)
        H.check_decode(out.cpu().numpy()[0].astype(np.float64), _ref("kvarn3", k, v, n, tail, q[0], hkv),
                       f"step {step}")
    assert c.status() == 0

