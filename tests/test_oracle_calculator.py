"""The pages' worked KV-size arithmetic (tests/golden/calculator_pins.txt), checked
against the oracle's calculator and against the library's host-only kvq_payload_bytes."""
import os

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
GIB = 2.0**30


def rows():
    out = []
    with open(os.path.join(HERE, "golden", "calculator_pins.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            c = [x.strip() for x in line.split("|")]
            out.append(dict(name=c[0], type=c[1], raw_bits=int(c[2]), layers=int(c[3]), heads=int(c[4]),
                            n=int(c[5]), tail=int(c[6]), want=float(c[7]), unit=c[8], tol=float(c[9])))
    return out


def _check(got_bytes, r):
    got = got_bytes / GIB if r["unit"] == "GiB" else got_bytes
    if r["tol"] == 0:
        assert got == r["want"], (r["name"], got)
    else:
        assert abs(got / r["want"] - 1) <= r["tol"], (r["name"], got)


@pytest.mark.parametrize("r", rows(), ids=lambda r: r["name"])
def test_oracle_calculator(r):
    _check(oracle.payload_bytes(r["type"], r["layers"], r["heads"], r["n"], r["tail"], raw_bits=r["raw_bits"]), r)


def test_q6_saves_20_to_25_percent_vs_q8():
    # BeeLLama.cpp v0.4.0 page, "Extended palette": q6_0/q6_1 save 20-25 % against q8_0
    saving = 1 - oracle.payload_bytes("q6_0", 1, 1, 1000, 0) / oracle.payload_bytes("q8_0", 1, 1, 1000, 0)
    assert 0.20 <= saving <= 0.25


def test_bits_per_value_of_the_palette():
    # same section: q2 "2.0-2.5", q3 "3.0-3.5", q6 "6.0-6.5" bits per value (qb_0 forms)
    for t, lo, hi in (("q2_0", 2.0, 2.5), ("q3_0", 3.0, 3.5), ("q6_0", 6.0, 6.5)):
        bpv = oracle.token_bytes(t) * 8 / 128
        assert lo <= bpv <= hi
