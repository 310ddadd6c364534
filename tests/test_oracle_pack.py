"""Pins of the packed code layout (the pages fix none; oracle/kvq_oracle.c, "packing",
defines it).  An independent unpacker written from the same definition, plus byte images
worked out by hand (tests/golden/pack_examples.txt)."""
import os

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
PLANES = {2: (2, 0), 3: (2, 1), 4: (4, 0), 5: (4, 1), 6: (4, 2), 8: (8, 0)}


def unpack_k_token(img, bits):
    """fields of the 128 channels of one K token image (16*bits bytes)"""
    img = [int(b) for b in img]
    wlo, whi = PLANES[bits]
    out = [0] * 128
    off = 0
    for w, shift in ((wlo, 0), (whi, wlo)):
        if w == 0:
            continue
        F = 8 // w
        for ch in range(128):
            blk, e = divmod(ch, 32)
            jj, k = divmod(e, 4)
            m, s = divmod(jj, F)
            byte = img[off + 16 * m + 4 * blk + k]
            out[ch] |= ((byte >> (s * w)) & ((1 << w) - 1)) << shift
        off += 16 * w
    return out


def unpack_v_quad(img, bits):
    """fields [4 tokens][128 channels] of one V quad image (64*bits bytes)"""
    img = [int(b) for b in img]
    wlo, whi = PLANES[bits]
    out = [[0] * 128 for _ in range(4)]
    off = 0
    for w, shift in ((wlo, 0), (whi, wlo)):
        if w == 0:
            continue
        F = 8 // w
        for k in range(4):
            for ch in range(128):
                blk, e = divmod(ch, 32)
                m, s = divmod(e, F)
                byte = img[off + 16 * w * blk + 4 * m + k]
                out[k][ch] |= ((byte >> (s * w)) & ((1 << w) - 1)) << shift
        off += 64 * w
    return out


def signed(f, bits):
    return f - (1 << bits) if f >= 1 << (bits - 1) else f


def _state(bits, n, seed, kvarn=False):
    rng = np.random.default_rng(seed)
    lo, hi = -(2 ** (bits - 1)), 2 ** (bits - 1)
    st = {
        "Q": n,
        "codes": rng.integers(lo, hi, (n, 128)).astype(np.int16),
        "d16": rng.integers(0, 0x7bff, (n, 4)).astype(np.uint16),
        "m16": rng.integers(0, 0x7bff, (n, 4)).astype(np.uint16),
        "t16": rng.integers(0x400, 0x7bff, n).astype(np.uint16),
        "c16": rng.integers(0x400, 0x7bff, (max(1, (n + 255) // 256), 128)).astype(np.uint16),
    }
    return st


@pytest.mark.parametrize("tname,bits", [("q2_0", 2), ("q3_0", 3), ("q4_0", 4), ("q5_0", 5), ("q6_0", 6),
                                        ("q8_0", 8), ("kvarn3", 3), ("q4_1", 4)])
@pytest.mark.parametrize("n_valid", [256, 7, 1])
def test_unpack_recovers_codes_and_scales(tname, bits, n_valid):
    st = _state(bits, n_valid, bits * 31 + n_valid)
    if tname.endswith("_1"):
        st["codes"] = (st["codes"].astype(np.int32) + 2 ** (bits - 1)).astype(np.int16)
    fam = oracle.family(tname)
    cb = 16 * bits
    for which in (0, 1):
        img, mask = oracle.pack_subpage(tname, which, st, 0)
        assert len(img) == oracle.subpage_bytes(tname)
        for i in range(n_valid):
            if which == 0:
                f = unpack_k_token(img[i * cb:(i + 1) * cb], bits)
            else:
                q, k = divmod(i, 4)
                f = unpack_v_quad(img[q * 4 * cb:(q + 1) * 4 * cb], bits)[k]
            vals = f if fam == 2 else [signed(x, bits) for x in f]
            assert vals == st["codes"][i].tolist()
        d_off = 256 * cb
        d = np.frombuffer(img[d_off:d_off + 2048].tobytes(), np.uint16).reshape(256, 4)
        assert np.array_equal(d[:n_valid], st["d16"][:n_valid])
        off = d_off + 2048
        if fam == 2:
            m = np.frombuffer(img[off:off + 2048].tobytes(), np.uint16).reshape(256, 4)
            assert np.array_equal(m[:n_valid], st["m16"][:n_valid])
            off += 2048
        if fam == 3:
            t = np.frombuffer(img[off:off + 512].tobytes(), np.uint16)
            assert np.array_equal(t[:n_valid], st["t16"][:n_valid])
            c = np.frombuffer(img[off + 512:off + 768].tobytes(), np.uint16)
            assert np.array_equal(c, st["c16"][0])
        # the mask marks the valid tokens' code bytes exactly
        if which == 0:
            assert mask[:n_valid * cb].all() and not mask[n_valid * cb:256 * cb].any()
        else:
            cm = mask[:256 * cb].reshape(64, 4 * cb)
            for i in range(256):
                q, k = divmod(i, 4)
                assert bool(cm[q, k::4].all()) == (i < n_valid)
                assert bool(cm[q, k::4].any()) == (i < n_valid)


def _golden():
    rows = {}
    with open(os.path.join(HERE, "golden", "pack_examples.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, bits, token, hexes = (x.strip() for x in line.split("|"))
            rows[name] = (int(bits), int(token), bytes.fromhex(hexes.replace(" ", "")))
    return rows


def test_hand_worked_images():
    g = _golden()
    bits, _, want = g["K4"]
    st = _state(4, 1, 0)
    st["codes"][:] = 0
    st["codes"][0, :32] = (np.arange(32) % 16) - 8
    img, _ = oracle.pack_subpage("q4_0", 0, st, 0)
    assert img[:64].tobytes() == want
    bits, tok, want = g["V2"]
    st = _state(2, 4, 0)
    st["codes"][:] = 0
    st["codes"][tok, 0] = 1
    st["codes"][tok, 5] = -1
    img, _ = oracle.pack_subpage("q2_0", 1, st, 0)
    assert img[:128].tobytes() == want
