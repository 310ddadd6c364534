"""ctypes binding of libkvq.so: the entry points of include/kvq.h under the same names.

Argument marshalling only (tensor -> pointer, Python ints -> C arrays); every step of
the append / decode / dequant path runs in the library's CUDA kernels.  The library is
loaded at import and a missing library is an ImportError: there is no fallback path.
"""
import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkvq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing; build it with `python -m bit_kv_cache_17_b200.build`")
_lib = C.CDLL(LIB_PATH)

# kvq_type (include/kvq.h)
TYPES = {
    "bf16": 0, "q2_0": 1, "q3_0": 2, "q4_0": 3, "q5_0": 4, "q6_0": 5, "q8_0": 6, "q4_1": 7,
    "kvarn2": 8, "kvarn3": 9, "kvarn4": 10, "kvarn5": 11, "kvarn6": 12, "kvarn8": 13,
    "q2_1": 14, "q3_1": 15, "q5_1": 16, "q6_1": 17,
}
KVQ_OK, KVQ_E_INVAL, KVQ_E_UNSUPPORTED, KVQ_E_CAPACITY = 0, -1, -2, -3
KVQ_E_ALIGN, KVQ_E_CUDA, KVQ_E_DEVICE, KVQ_E_SIZE = -4, -5, -6, -7


class kvq_params(C.Structure):
    _fields_ = [
        ("n_layers", C.c_int32), ("n_seqs", C.c_int32), ("n_kv_heads", C.c_int32),
        ("head_dim", C.c_int32), ("max_ctx", C.c_int64), ("type_k", C.c_int32),
        ("type_v", C.c_int32), ("tail", C.c_int32), ("group", C.c_int32),
        ("sinkhorn_iters", C.c_int32), ("page_tokens", C.c_int32), ("var_norm", C.c_int32), ("tail_f16", C.c_int32),
    ]


class KVQError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {kvq_strerror(code)} ({code})")


_vp, _i32, _i64, _sz = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t
_SIG = {
    "kvq_default_params": (None, [C.POINTER(kvq_params)]),
    "kvq_cache_bytes": (C.c_int, [C.POINTER(kvq_params), C.POINTER(_sz)]),
    "kvq_payload_bytes": (C.c_int, [_i32, _i32, _i64, _i64, _i64, _i64, C.POINTER(C.c_double)]),
    "kvq_cache_create": (C.c_int, [C.POINTER(kvq_params), _vp, _sz, C.POINTER(_vp)]),
    "kvq_cache_destroy": (None, [_vp]),
    "kvq_append": (C.c_int, [_vp, _i32, _i32, C.POINTER(_i32), C.POINTER(_i32), _vp, _vp, _vp]),
    "kvq_workspace_bytes": (C.c_int, [_vp, _i32, _i32, C.POINTER(_sz)]),
    "kvq_decode_attn": (C.c_int, [_vp, _i32, _i32, C.POINTER(_i32), _i32, _vp, C.c_float, _vp, _vp, _sz, _vp]),
    "kvq_prefill_attn": (C.c_int, [_vp, _i32, _i32, _i32, _i32, _vp, C.c_float, _vp, _vp, _sz, _vp]),
    "kvq_append_decode": (C.c_int, [_vp, _i32, _i32, C.POINTER(_i32), C.POINTER(_i32), _vp, _vp, _i32, _vp,
                                    C.c_float, _vp, _vp, _sz, _vp]),
    "kvq_dequant": (C.c_int, [_vp, _i32, _i32, _i32, _i64, _i64, _i32, _vp, _vp]),
    "kvq_seq_len": (C.c_int, [_vp, _i32, _i32, C.POINTER(_i64)]),
    "kvq_seq_reset": (C.c_int, [_vp, _i32]),
    "kvq_locate": (C.c_int, [_vp, _i32, _i32, _i32, _i64, _i32, _i32, _i64, C.POINTER(_sz), C.POINTER(_sz)]),
    "kvq_get_status": (C.c_int, [_vp, _vp]),
    "kvq_describe": (C.c_char_p, [_vp]),
    "kvq_strerror": (C.c_char_p, [C.c_int]),
    "kvq_launch_count": (C.c_int, [C.POINTER(C.c_uint64)]),
    "kvq_decode_attn_noalloc": (C.c_int, [_vp, _i32, _i32, C.POINTER(_i32), _i32, _vp, C.c_float, _vp, _vp]),
}
for _name, (_res, _args) in _SIG.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_SIG)


def _check(rc, where):
    if rc != KVQ_OK:
        raise KVQError(rc, where)


def _i32arr(xs):
    xs = [int(x) for x in xs]
    return (_i32 * max(1, len(xs)))(*xs)


def kvq_strerror(code):
    return _lib.kvq_strerror(code).decode()


def kvq_default_params(**overrides):
    p = kvq_params()
    _lib.kvq_default_params(C.byref(p))
    for k, v in overrides.items():
        if k in ("type_k", "type_v") and isinstance(v, str):
            v = TYPES[v]
        setattr(p, k, v)
    return p


def kvq_cache_bytes(p):
    n = _sz()
    _check(_lib.kvq_cache_bytes(C.byref(p), C.byref(n)), "kvq_cache_bytes")
    return n.value


def kvq_payload_bytes(type_, n_layers, n_kv_heads, n, tail, raw_bits=0):
    t = TYPES[type_] if isinstance(type_, str) else int(type_)
    out = C.c_double()
    _check(_lib.kvq_payload_bytes(t, raw_bits, n_layers, n_kv_heads, n, tail, C.byref(out)), "kvq_payload_bytes")
    return out.value


def kvq_cache_create(p, dev_ptr, nbytes):
    h = _vp()
    _check(_lib.kvq_cache_create(C.byref(p), _vp(dev_ptr), nbytes, C.byref(h)), "kvq_cache_create")
    return h


def kvq_cache_destroy(h):
    _lib.kvq_cache_destroy(h)


def kvq_append(h, layer, seq_ids, n_new, k_ptr, v_ptr, stream=0):
    rc = _lib.kvq_append(h, layer, len(seq_ids), _i32arr(seq_ids), _i32arr(n_new), _vp(k_ptr), _vp(v_ptr), _vp(stream))
    _check(rc, "kvq_append")


def kvq_workspace_bytes(h, n_seqs, n_q_heads):
    n = _sz()
    _check(_lib.kvq_workspace_bytes(h, n_seqs, n_q_heads, C.byref(n)), "kvq_workspace_bytes")
    return n.value


def kvq_decode_attn(h, layer, seq_ids, n_q_heads, q_ptr, softmax_scale, out_ptr, ws_ptr, ws_bytes, stream=0):
    rc = _lib.kvq_decode_attn(h, layer, len(seq_ids), _i32arr(seq_ids), n_q_heads, _vp(q_ptr), softmax_scale,
                              _vp(out_ptr), _vp(ws_ptr), ws_bytes, _vp(stream))
    _check(rc, "kvq_decode_attn")


def kvq_append_decode(h, layer, seq_ids, n_new, k_ptr, v_ptr, n_q_heads, q_ptr, softmax_scale, out_ptr, ws_ptr,
                      ws_bytes, stream=0):
    rc = _lib.kvq_append_decode(h, layer, len(seq_ids), _i32arr(seq_ids), _i32arr(n_new), _vp(k_ptr), _vp(v_ptr),
                                n_q_heads, _vp(q_ptr), softmax_scale, _vp(out_ptr), _vp(ws_ptr), ws_bytes, _vp(stream))
    _check(rc, "kvq_append_decode")


def kvq_prefill_attn(h, layer, seq, n_q_tokens, n_q_heads, q_ptr, softmax_scale, out_ptr, ws_ptr, ws_bytes, stream=0):
    rc = _lib.kvq_prefill_attn(h, layer, seq, n_q_tokens, n_q_heads, _vp(q_ptr), softmax_scale, _vp(out_ptr),
                               _vp(ws_ptr), ws_bytes, _vp(stream))
    _check(rc, "kvq_prefill_attn")


def kvq_decode_attn_noalloc(h, layer, seq_ids, n_q_heads, q_ptr, softmax_scale, out_ptr, stream=0):
    rc = _lib.kvq_decode_attn_noalloc(h, layer, len(seq_ids), _i32arr(seq_ids), n_q_heads, _vp(q_ptr), softmax_scale,
                                      _vp(out_ptr), _vp(stream))
    _check(rc, "kvq_decode_attn_noalloc")


def kvq_dequant(h, layer, seq, which, t0, t1, basis, out_ptr, stream=0):
    _check(_lib.kvq_dequant(h, layer, seq, which, t0, t1, basis, _vp(out_ptr), _vp(stream)), "kvq_dequant")


def kvq_seq_len(h, layer, seq):
    n = _i64()
    _check(_lib.kvq_seq_len(h, layer, seq, C.byref(n)), "kvq_seq_len")
    return n.value


def kvq_seq_reset(h, seq):
    _check(_lib.kvq_seq_reset(h, seq), "kvq_seq_reset")


def kvq_locate(h, kind, layer, seq, page, head, which, token=0):
    off, nb = _sz(), _sz()
    _check(_lib.kvq_locate(h, kind, layer, seq, page, head, which, token, C.byref(off), C.byref(nb)), "kvq_locate")
    return off.value, nb.value


def kvq_get_status(h, stream=0):
    return _lib.kvq_get_status(h, _vp(stream))


def kvq_launch_count():
    n = C.c_uint64()
    _check(_lib.kvq_launch_count(C.byref(n)), "kvq_launch_count")
    return n.value


def kvq_describe(h):
    return _lib.kvq_describe(h).decode()


class KVCache:
    """A cache whose storage and workspace are torch tensors on one CUDA device.

    PyTorch supplies the device memory and the stream; every call goes straight to the
    C ABI with the tensors' pointers.
    """

    def __init__(self, device=None, **params):
        import torch

        self.torch = torch
        self.params = kvq_default_params(**params)
        self.nbytes = kvq_cache_bytes(self.params)
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.storage = torch.empty(self.nbytes, dtype=torch.uint8, device=self.device)
        with torch.cuda.device(self.device):
            self.handle = kvq_cache_create(self.params, self.storage.data_ptr(), self.nbytes)
        self._ws = None
        self._ws_bytes = {}  # (n_seqs, n_q_heads) -> kvq_workspace_bytes

    def __del__(self):
        h = getattr(self, "handle", None)
        if h:
            kvq_cache_destroy(h)
            self.handle = None

    def _stream(self, stream):
        if stream is None:
            stream = self.torch.cuda.current_stream(self.device)
        return stream.cuda_stream

    def append(self, layer, seq_ids, n_new, k, v, stream=None):
        assert k.dtype == self.torch.bfloat16 and v.dtype == self.torch.bfloat16
        assert k.is_contiguous() and v.is_contiguous()
        kvq_append(self.handle, layer, list(seq_ids), list(n_new), k.data_ptr(), v.data_ptr(), self._stream(stream))

    def workspace(self, n_seqs, n_q_heads):
        key = (n_seqs, n_q_heads)
        nb = self._ws_bytes.get(key)
        if nb is None:
            nb = self._ws_bytes[key] = kvq_workspace_bytes(self.handle, n_seqs, n_q_heads)
        if self._ws is None or self._ws.numel() < nb:
            self._ws = self.torch.empty(max(nb, 256), dtype=self.torch.uint8, device=self.device)
        return self._ws

    def decode(self, layer, seq_ids, q, out=None, softmax_scale=0.0, stream=None):
        assert q.dtype == self.torch.float32 and q.is_contiguous()
        n_seqs, n_q_heads = q.shape[0], q.shape[1]
        if out is None:
            out = self.torch.empty_like(q)
        ws = self.workspace(n_seqs, n_q_heads)
        kvq_decode_attn(self.handle, layer, list(seq_ids), n_q_heads, q.data_ptr(), softmax_scale, out.data_ptr(),
                        ws.data_ptr(), ws.numel(), self._stream(stream))
        return out

    def append_decode(self, layer, seq_ids, n_new, k, v, q, out=None, softmax_scale=0.0, stream=None):
        """kvq_append_decode: append n_new[i] rows to seq_ids[i], then decode q (row i for
        seq_ids[i]) over the grown cache, the decode overlapping the append."""
        assert k.dtype == self.torch.bfloat16 and v.dtype == self.torch.bfloat16
        assert k.is_contiguous() and v.is_contiguous()
        assert q.dtype == self.torch.float32 and q.is_contiguous()
        n_seqs, n_q_heads = q.shape[0], q.shape[1]
        if out is None:
            out = self.torch.empty_like(q)
        ws = self.workspace(n_seqs, n_q_heads)
        kvq_append_decode(self.handle, layer, list(seq_ids), list(n_new), k.data_ptr(), v.data_ptr(), n_q_heads,
                          q.data_ptr(), softmax_scale, out.data_ptr(), ws.data_ptr(), ws.numel(), self._stream(stream))
        return out

    def prefill_attn(self, layer, seq, q, out=None, softmax_scale=0.0, stream=None):
        """kvq_prefill_attn: q [n_q_tokens, n_q_heads, 128] fp32, causal over the chunk of the
        sequence's newest n_q_tokens tokens."""
        assert q.dtype == self.torch.float32 and q.is_contiguous()
        n_q, n_q_heads = q.shape[0], q.shape[1]
        if out is None:
            out = self.torch.empty_like(q)
        ws = self.workspace(n_q, n_q_heads)
        kvq_prefill_attn(self.handle, layer, seq, n_q, n_q_heads, q.data_ptr(), softmax_scale, out.data_ptr(),
                         ws.data_ptr(), ws.numel(), self._stream(stream))
        return out

    def dequant(self, layer, seq, which, t0, t1, basis=0, out=None, stream=None):
        if out is None:
            out = self.torch.empty((t1 - t0, self.params.n_kv_heads, 128), dtype=self.torch.float32, device=self.device)
        kvq_dequant(self.handle, layer, seq, which, t0, t1, basis, out.data_ptr(), self._stream(stream))
        return out

    def seq_len(self, layer, seq):
        return kvq_seq_len(self.handle, layer, seq)

    def reset(self, seq):
        kvq_seq_reset(self.handle, seq)

    def locate(self, kind, layer, seq, page, head, which, token=0):
        return kvq_locate(self.handle, kind, layer, seq, page, head, which, token)

    def status(self, stream=None):
        return kvq_get_status(self.handle, self._stream(stream))

    def describe(self):
        return kvq_describe(self.handle)
