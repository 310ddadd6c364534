"""The C-ABI library loads without a GPU, exports every entry point include/kvq.h
declares, and validates arguments on the host (no device call is needed for these)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared():
    src = open(os.path.join(ROOT, "include", "kvq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    from bit_kv_cache_17_b200 import kvq

    lib = C.CDLL(kvq.LIB_PATH)
    names = declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(kvq.EXPORTED)


def test_host_validation_and_sizes():
    from bit_kv_cache_17_b200 import kvq

    p = kvq.kvq_default_params(n_kv_heads=8, max_ctx=65536, type_k="kvarn4", type_v="kvarn4", tail=1024)
    nb = kvq.kvq_cache_bytes(p)
    # 256 pages x 8 heads x (K + V sub-pages of 19200 B) plus a 1280-row ring per stream
    assert nb >= 256 * 8 * 2 * 19200 + 8 * 2 * 1280 * 256
    for bad in (dict(head_dim=64), dict(group=128), dict(page_tokens=512)):
        with pytest.raises(kvq.KVQError) as e:
            kvq.kvq_cache_bytes(kvq.kvq_default_params(**bad))
        assert e.value.code == kvq.KVQ_E_UNSUPPORTED
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_cache_bytes(kvq.kvq_default_params(type_k="bf16", type_v="q4_0"))
    assert e.value.code == kvq.KVQ_E_UNSUPPORTED
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_cache_bytes(kvq.kvq_default_params(tail=-1))
    assert e.value.code == kvq.KVQ_E_INVAL
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_cache_create(p, 0, nb)
    assert e.value.code == kvq.KVQ_E_INVAL
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_cache_create(p, 8, nb)  # misaligned pointer is rejected before any device call
    assert e.value.code == kvq.KVQ_E_ALIGN
    assert kvq.kvq_strerror(kvq.KVQ_E_CAPACITY).startswith("sequence capacity")


def test_var_norm_resolves_to_the_kvarn_type():
    """The pages' --cache-var-norm switch: qN_0 with KVarN normalization is kvarnN (same
    rotation, balancing and symmetric quantizer); qN_1 and BF16 have no such form."""
    from bit_kv_cache_17_b200 import kvq

    for b in (2, 3, 4, 5, 6, 8):
        a = kvq.kvq_cache_bytes(kvq.kvq_default_params(type_k=f"q{b}_0", type_v=f"q{b}_0", var_norm=1))
        r = kvq.kvq_cache_bytes(kvq.kvq_default_params(type_k=f"kvarn{b}", type_v=f"kvarn{b}"))
        assert a == r
    assert kvq.kvq_cache_bytes(kvq.kvq_default_params(type_k="kvarn4", type_v="kvarn4", var_norm=1)) == \
        kvq.kvq_cache_bytes(kvq.kvq_default_params(type_k="kvarn4", type_v="kvarn4"))
    for t in ("q4_1", "bf16"):
        with pytest.raises(kvq.KVQError) as e:
            kvq.kvq_cache_bytes(kvq.kvq_default_params(type_k=t, type_v=t, var_norm=1))
        assert e.value.code == kvq.KVQ_E_UNSUPPORTED
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_cache_bytes(kvq.kvq_default_params(var_norm=2))
    assert e.value.code == kvq.KVQ_E_INVAL


def test_tail_format_flag():
    """tail_f16 takes 0 (BF16 tail) or 1 (F16 tail); the tail format does not change sizes."""
    from bit_kv_cache_17_b200 import kvq

    a = kvq.kvq_cache_bytes(kvq.kvq_default_params(tail_f16=0))
    assert kvq.kvq_cache_bytes(kvq.kvq_default_params(tail_f16=1)) == a
    with pytest.raises(kvq.KVQError) as e:
        kvq.kvq_cache_bytes(kvq.kvq_default_params(tail_f16=2))
    assert e.value.code == kvq.KVQ_E_INVAL
