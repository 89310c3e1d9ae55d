"""Checks on the seeded input generator (data recipe only)."""
import math

import numpy as np

from any_precision_expert_pw_b200.inputs import (CONFIGS, MIN_BITS, f32_to_bf16_bits,
                                                 make_layer, nested_luts)


def test_bf16_rounding_is_rne():
    a = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, -2.5, 1.0 + 2**-8 + 2**-20], np.float32)
    bits = f32_to_bf16_bits(a)
    assert bits.tolist() == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x3F81]


def test_nested_luts_sorted_and_nested():
    rng = np.random.default_rng(0)
    parent = np.sort(rng.normal(0, 0.02, size=(9, 256)).astype(np.float16), axis=1)
    luts = nested_luts(parent, 8)
    assert sorted(luts) == list(range(MIN_BITS, 9))
    for b, t in luts.items():
        assert t.shape == (9, 1 << b) and t.dtype == np.float16
        assert (np.diff(t.astype(np.float64), axis=1) >= 0).all()
        g = 1 << (8 - b)
        grp = parent.astype(np.float64).reshape(9, 1 << b, g)
        assert (t >= grp.min(axis=2)).all() and (t <= grp.max(axis=2)).all()


def test_tiny_layer_recipe():
    cfg = CONFIGS["tiny"]
    L = make_layer(cfg, 4)
    assert L.q.shape == (8, 2) and set(np.unique(L.q)) <= {3, 4}
    assert L.idx[0][0].shape == (1024, 256) and L.idx[0][1].shape == (256, 512)
    assert L.idx[0][0].max() < 16
    assert L.x_bf16.shape == (4, 256) and L.resident is None and not L.bias.any()
    L2 = make_layer(cfg, 4)
    assert np.array_equal(L.idx[5][1], L2.idx[5][1]) and np.array_equal(L.x_bf16, L2.x_bf16)


def test_zipf_bias_and_residency():
    L = make_layer(CONFIGS["mixtral_8x7b"], 1, with_weights=False)
    rho = np.sort(np.exp(L.bias.astype(np.float64)))[::-1]
    j = np.arange(1, 9)
    want = j ** -1.2 / (j ** -1.2).sum()
    assert np.allclose(rho, want, rtol=1e-6)
    R = make_layer(CONFIGS["qwen3_next_80b_a3b"], 16, with_weights=False)
    assert int(R.resident.sum()) == math.floor(0.25 * 512)
