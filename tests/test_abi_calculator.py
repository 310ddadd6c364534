"""The library's host-only calculator (kvq_payload_bytes) against the pages' worked
arithmetic in tests/golden/calculator_pins.txt."""
import pytest

from test_oracle_calculator import _check, rows


@pytest.mark.parametrize("r", rows(), ids=lambda r: r["name"])
def test_library_calculator(r):
    from bit_kv_cache_17_b200 import kvq

    _check(kvq.kvq_payload_bytes(r["type"], r["layers"], r["heads"], r["n"], r["tail"], raw_bits=r["raw_bits"]), r)


def test_q6_saves_20_to_25_percent_vs_q8():
    # BeeLLama.cpp v0.4.0 page, "Extended palette": q6_0/q6_1 save 20-25 % against q8_0
    from bit_kv_cache_17_b200 import kvq

    saving = 1 - kvq.kvq_payload_bytes("q6_0", 1, 1, 1000, 0) / kvq.kvq_payload_bytes("q8_0", 1, 1, 1000, 0)
    assert 0.20 <= saving <= 0.25
