"""kvq_dequant vs the oracle's fp64 dequantization of the same (bit-exact) state."""
import numpy as np
import pytest

import gpu_helpers as H
import oracle
from bit_kv_cache_17_b200 import synth


pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("t", ["kvarn4", "kvarn6", "q5_0", "q3_1", "bf16"])
def test_dequant_matches_oracle(t):
    hkv, n, tail = 2, 700, 150
    rng = np.random.default_rng(3)
    k, v, _ = synth.kv_ar1(rng, hkv, n)
    c = H.make_cache(t, hkv, 1024, tail)
    H.append(c, 0, [0], [(synth.token_major(k), synth.token_major(v))])
    for which, hist in ((0, k), (1, v)):
        for basis in (0, 1):
            got = c.dequant(0, 0, which, 0, n, basis=basis).cpu().numpy()  # [n, hkv, 128]
            for h in range(hkv):
                if t == "bf16":
                    ref = synth.bf16_to_f32(hist[h]).astype(np.float64)
                    assert np.array_equal(got[:, h].astype(np.float64), ref)
                    continue
                st = oracle.stream_state(t, hist[h], tail)
                Q = st["Q"]
                ref = oracle.dequant(t, st, basis=basis)
                scale = np.abs(ref).max()
                assert np.max(np.abs(got[:Q, h] - ref)) <= 2e-6 * scale
                # tail rows come back exactly
                assert np.array_equal(got[Q:, h], synth.bf16_to_f32(hist[h][Q:]))
    sub = c.dequant(0, 0, 1, 123, 456, basis=0).cpu().numpy()
    full = c.dequant(0, 0, 1, 0, n, basis=0).cpu().numpy()
    assert np.array_equal(sub, full[123:456])
