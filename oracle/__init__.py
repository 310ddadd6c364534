"""CPU oracle for the mixed-precision KV cache - TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py (its cpu_baseline leg and its
``--impl reference`` arm) may import this package.  It wraps the plain C oracle in
kvq_oracle.c (built by oracle/build.py with gcc) through ctypes and never touches the
CUDA library.  Every function cites, in kvq_oracle.c, the page passage it follows.
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

_LIB = None

TYPES = {
    "bf16": 0, "q2_0": 1, "q3_0": 2, "q4_0": 3, "q5_0": 4, "q6_0": 5, "q8_0": 6, "q4_1": 7,
    "kvarn2": 8, "kvarn3": 9, "kvarn4": 10, "kvarn5": 11, "kvarn6": 12, "kvarn8": 13,
    "q2_1": 14, "q3_1": 15, "q5_1": 16, "q6_1": 17,
}
D = 128
GROUP = 256

_i32, _i64, _f32, _f64, _p = C.c_int, C.c_int64, C.c_float, C.c_double, C.c_void_p


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = C.CDLL(path)
        sig = {
            "kvqo_type_family": (_i32, [_i32]),
            "kvqo_type_bits": (_i32, [_i32]),
            "kvqo_token_bytes": (_i32, [_i32]),
            "kvqo_subpage_bytes": (_i32, [_i32]),
            "kvqo_f32_to_bf16_n": (None, [_p, _p, _i64]),
            "kvqo_f32_to_f16_n": (None, [_p, _p, _i64]),
            "kvqo_f16_to_f32_n": (None, [_p, _p, _i64]),
            "kvqo_wht128": (None, [_p]),
            "kvqo_wht128_f64": (None, [_p]),
            "kvqo_sinkhorn": (None, [_p, _i32, _i32, _p, _p]),
            "kvqo_sinkhorn_literal": (None, [_p, _i32, _i32, _p, _p]),
            "kvqo_quant_sym": (None, [_p, _i32, _p, _p]),
            "kvqo_quant_asym": (None, [_p, _i32, _p, _p, _p]),
            "kvqo_stream_state": (_i64, [_i32, _p, _i64, _i64, _i32, _p, _p, _p, _p, _p]),
            "kvqo_pack_subpage": (_i32, [_i32, _i32, _i32, _p, _p, _p, _p, _p, _p, _p]),
            "kvqo_dequant": (_i32, [_i32, _i64, _p, _p, _p, _p, _p, _i32, _p]),
            "kvqo_attend": (None, [_p, _i32, _p, _p, _i64, _f64, _p]),
            "kvqo_decode_head": (_i32, [_i32, _i32, _p, _p, _i64, _i64, _i32, _p, _i32, _f64, _p]),
            "kvqo_prefill_head": (_i32, [_i32, _i32, _p, _p, _i64, _i64, _i32, _p, _i32, _i32, _f64, _p]),
            "kvqo_payload_bytes": (_f64, [_i32, _i32, _i64, _i64, _i64, _i64, _i64]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def _tid(t):
    return TYPES[t] if isinstance(t, str) else int(t)


def _ptr(a):
    return a.ctypes.data_as(C.c_void_p) if a is not None else None


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def family(t):
    return lib().kvqo_type_family(_tid(t))


def bits(t):
    return lib().kvqo_type_bits(_tid(t))


def token_bytes(t):
    return lib().kvqo_token_bytes(_tid(t))


def subpage_bytes(t):
    return lib().kvqo_subpage_bytes(_tid(t))


def f32_to_bf16(x):
    x = _c(x, np.float32)
    y = np.empty(x.shape, np.uint16)
    lib().kvqo_f32_to_bf16_n(_ptr(x), _ptr(y), x.size)
    return y


def bf16_to_f32(h):
    h = _c(h, np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)


def f32_to_f16(x):
    x = _c(x, np.float32)
    y = np.empty(x.shape, np.uint16)
    lib().kvqo_f32_to_f16_n(_ptr(x), _ptr(y), x.size)
    return y


def f16_to_f32(h):
    h = _c(h, np.uint16)
    y = np.empty(h.shape, np.float32)
    lib().kvqo_f16_to_f32_n(_ptr(h), _ptr(y), h.size)
    return y


def f16_tail_bits(x_bf16):
    """The F16 tail's stored value of each BF16 input ("KV Cache Precision Tail": the newest
    tokens stay 16-bit, BF16 or F16): fp16 round to nearest even, overflow to inf."""
    return f32_to_f16(bf16_to_f32(x_bf16))


def f16_tail_rows(x_bf16):
    """The values a stream with an F16 tail holds and quantizes, as BF16 bits.  Every fp16
    rounding of a BF16 value is again a BF16 value (checked here), so that stream is the
    BF16-tail stream of these rows."""
    y = f16_to_f32(f16_tail_bits(x_bf16))
    b = f32_to_bf16(y)
    back = bf16_to_f32(b)
    assert np.array_equal(back[~np.isnan(y)], y[~np.isnan(y)])
    return b


def wht128(v):
    v = _c(v, np.float32).copy()
    assert v.shape[-1] == D
    for row in v.reshape(-1, D):
        lib().kvqo_wht128(_ptr(row))
    return v


def wht128_f64(v):
    v = _c(v, np.float64).copy()
    for row in v.reshape(-1, D):
        lib().kvqo_wht128_f64(_ptr(row))
    return v


def sinkhorn(x, iters=8):
    x = _c(x, np.float32)
    n = x.shape[0]
    c = np.empty(D, np.float32)
    t = np.empty(n, np.float32)
    lib().kvqo_sinkhorn(_ptr(x), n, iters, _ptr(c), _ptr(t))
    return c, t


def sinkhorn_literal(x, iters=8):
    x = _c(x, np.float64)
    n = x.shape[0]
    c = np.empty(D, np.float64)
    t = np.empty(n, np.float64)
    lib().kvqo_sinkhorn_literal(_ptr(x), n, iters, _ptr(c), _ptr(t))
    return c, t


def quant_sym(y, nbits):
    y = _c(y, np.float32)
    d = np.zeros(1, np.uint16)
    codes = np.zeros(32, np.int16)
    lib().kvqo_quant_sym(_ptr(y), nbits, _ptr(d), _ptr(codes))
    return int(d[0]), codes


def quant_asym(x, nbits):
    x = _c(x, np.float32)
    d = np.zeros(1, np.uint16)
    m = np.zeros(1, np.uint16)
    codes = np.zeros(32, np.int16)
    lib().kvqo_quant_asym(_ptr(x), nbits, _ptr(d), _ptr(m), _ptr(codes))
    return int(d[0]), int(m[0]), codes


def stream_state(t, x_bf16, tail, iters=8):
    """State of the quantized region of one stream from its BF16 history (n x 128)."""
    x = _c(x_bf16, np.uint16).reshape(-1, D)
    n = x.shape[0]
    Q = max(n - min(n, tail), 0) if family(t) != 0 else 0
    ng = (Q + GROUP - 1) // GROUP
    st = {
        "Q": Q,
        "codes": np.zeros((Q, D), np.int16),
        "d16": np.zeros((Q, 4), np.uint16),
        "m16": np.zeros((Q, 4), np.uint16),
        "t16": np.zeros(Q, np.uint16),
        "c16": np.zeros((ng, D), np.uint16),
    }
    if n == 0:
        return st
    r = lib().kvqo_stream_state(_tid(t), _ptr(x), n, tail, iters, _ptr(st["codes"]), _ptr(st["d16"]),
                                _ptr(st["m16"]), _ptr(st["t16"]), _ptr(st["c16"]))
    assert r == Q, (r, Q)
    return st


def pack_subpage(t, which, st, page):
    """Byte image and valid-byte mask of page `page` (256 tokens) of a stream state."""
    nb = subpage_bytes(t)
    a = page * GROUP
    nv = max(0, min(GROUP, st["Q"] - a))
    img = np.zeros(nb, np.uint8)
    mask = np.zeros(nb, np.uint8)
    sl = slice(a, a + nv)
    codes = _c(st["codes"][sl], np.int16)
    d16 = _c(st["d16"][sl], np.uint16)
    m16 = _c(st["m16"][sl], np.uint16)
    t16 = _c(st["t16"][sl], np.uint16)
    c16 = _c(st["c16"][page] if st["c16"].shape[0] > page else np.zeros(D), np.uint16)
    r = lib().kvqo_pack_subpage(_tid(t), which, nv, _ptr(codes), _ptr(d16), _ptr(m16), _ptr(t16),
                                _ptr(c16), _ptr(img), _ptr(mask))
    assert r == nb
    return img, mask


def dequant(t, st, basis=0):
    Q = st["Q"]
    out = np.zeros((Q, D), np.float64)
    if Q == 0:
        return out
    r = lib().kvqo_dequant(_tid(t), Q, _ptr(_c(st["codes"], np.int16)), _ptr(_c(st["d16"], np.uint16)),
                           _ptr(_c(st["m16"], np.uint16)), _ptr(_c(st["t16"], np.uint16)),
                           _ptr(_c(st["c16"], np.uint16)), basis, _ptr(out))
    assert r == 0
    return out


def attend(q, k, v, scale):
    q = _c(q, np.float64).reshape(-1, D)
    k = _c(k, np.float64).reshape(-1, D)
    v = _c(v, np.float64).reshape(-1, D)
    out = np.zeros_like(q)
    lib().kvqo_attend(_ptr(q), q.shape[0], _ptr(k), _ptr(v), k.shape[0], scale, _ptr(out))
    return out


def decode_head(type_k, type_v, xk_bf16, xv_bf16, tail, q, scale=None, iters=8):
    """fp64 decode of G query rows (G x 128 fp32) against one KV head's full history."""
    xk = _c(xk_bf16, np.uint16).reshape(-1, D)
    xv = _c(xv_bf16, np.uint16).reshape(-1, D)
    q = _c(q, np.float32).reshape(-1, D)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.zeros((q.shape[0], D), np.float64)
    r = lib().kvqo_decode_head(_tid(type_k), _tid(type_v), _ptr(xk), _ptr(xv), xk.shape[0], tail, iters,
                               _ptr(q), q.shape[0], float(scale), _ptr(out))
    assert r == 0
    return out


def prefill_head(type_k, type_v, xk_bf16, xv_bf16, tail, q, scale=None, iters=8):
    """fp64 attention of a chunk of n_q queries (n_q x G x 128 fp32), the chunk being the n_q
    newest tokens of one KV head's history: query i sees rows [0, n - n_q + 1 + i) of the
    state of the full history."""
    xk = _c(xk_bf16, np.uint16).reshape(-1, D)
    xv = _c(xv_bf16, np.uint16).reshape(-1, D)
    q = _c(q, np.float32)
    n_q, G = q.shape[0], q.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.zeros((n_q, G, D), np.float64)
    r = lib().kvqo_prefill_head(_tid(type_k), _tid(type_v), _ptr(xk), _ptr(xv), xk.shape[0], tail, iters,
                                _ptr(q), n_q, G, float(scale), _ptr(out))
    assert r == 0
    return out


def payload_bytes(t, n_layers, n_kv_heads, n, tail, head_dim=D, raw_bits=0):
    return lib().kvqo_payload_bytes(_tid(t), raw_bits, n_layers, n_kv_heads, head_dim, n, tail)
