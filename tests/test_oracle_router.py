"""Pins for the oracle's router GEMV and softmax top-k (CPU only)."""
import itertools
import math

import numpy as np
import pytest

from any_precision_expert_pw_b200.inputs import f32_to_bf16_bits, random_router_inputs
from oracle.router import router_logits, softmax_topk


def _bf16(a):
    return f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def test_hand_built_one_hot_and_ties(golden):
    g = golden("router_hand.json")
    for case in ("A", "B"):
        c = g[case]
        x = _bf16([c["x"]])
        logits = router_logits(x, np.array(c["Wr"], np.float32), np.array(c["bias"], np.float32))
        assert logits[0].tolist() == c["logits"]
        idx, gate, _ = softmax_topk(logits, c["k"], renorm=True)
        assert idx[0].tolist() == c["idx"]
    # closed forms for case A
    l = g["A"]["logits"]
    Z = sum(math.exp(v) for v in l)
    idx, gate, g64 = softmax_topk(np.array([l], np.float32), 2, renorm=False)
    assert g64[0, 0] == pytest.approx(math.exp(0.5) / Z, rel=1e-14)
    assert g64[0, 1] == pytest.approx(math.exp(0.25) / Z, rel=1e-14)
    _, _, g64 = softmax_topk(np.array([l], np.float32), 2, renorm=True)
    assert g64[0, 0] == pytest.approx(1.0 / (1.0 + math.exp(-0.25)), rel=1e-14)
    assert g64[0, 1] == pytest.approx(1.0 / (1.0 + math.exp(0.25)), rel=1e-14)


def test_one_hot_rows_give_router_columns():
    x_bits, Wr, bias = random_router_inputs(1, 16, 64, seed=3, zipf_s=1.2)
    for c in (0, 17, 63):
        x = np.zeros((1, 64), np.float32)
        x[0, c] = 1.0
        logits = router_logits(_bf16(x), Wr, bias)
        assert np.array_equal(logits[0], (Wr[:, c].astype(np.float64) + bias).astype(np.float32))


def test_brute_force_topk_matches_all_subsets():
    # the chosen set maximises the logit sum; order within it is by logit then index
    rng = np.random.default_rng(0)
    for trial in range(30):
        E, k = int(rng.integers(2, 9)), 0
        k = int(rng.integers(1, E + 1))
        logits = np.round(rng.normal(size=(1, E)) * 2) / 2     # many ties
        logits = logits.astype(np.float32)
        idx, _, _ = softmax_topk(logits, k, renorm=False)
        best = None
        for comb in itertools.combinations(range(E), k):
            key = (sum(float(logits[0, e]) for e in comb), tuple(-e for e in comb))
            if best is None or key > best[0]:
                best = (key, comb)
        assert set(idx[0].tolist()) == set(best[1])
        vals = [(-float(logits[0, e]), e) for e in idx[0]]
        assert vals == sorted(vals)


def test_special_cases():
    logits = np.array([[0.5, -1.0, 2.0, 2.0, 0.0]], np.float32)
    idx, gate, g64 = softmax_topk(logits, 5, renorm=False)      # k = E: every expert, ordered
    assert idx[0].tolist() == [2, 3, 0, 4, 1]
    assert g64.sum() == pytest.approx(1.0, abs=1e-15)
    idx, gate, _ = softmax_topk(logits, 1, renorm=True)          # k = 1 with renorm: gate 1
    assert idx[0].tolist() == [2] and gate[0, 0] == 1.0
    eq = np.zeros((3, 6), np.float32)                              # all-equal logits
    idx, gate, g64 = softmax_topk(eq, 4, renorm=False)
    assert (idx == np.arange(4)).all() and np.allclose(g64, 1 / 6, rtol=0, atol=1e-16)
    idx, gate, g64 = softmax_topk(eq, 4, renorm=True)
    assert np.allclose(g64, 0.25, rtol=0, atol=1e-16)


def test_softmax_shift_invariance_and_two_expert_sigmoid():
    l = np.array([[1.25, -0.75]], np.float32)
    _, _, g = softmax_topk(l, 2, renorm=False)
    assert g[0, 0] == pytest.approx(1 / (1 + math.exp(-2.0)), rel=1e-14)
    _, _, g2 = softmax_topk(l + np.float32(3.0), 2, renorm=False)
    assert np.allclose(g, g2, rtol=1e-14, atol=0)


def test_logit_sum_within_dot_product_bound():
    # against an exactly rounded sum (math.fsum) of the exact products
    x_bits, Wr, bias = random_router_inputs(3, 5, 257, seed=4)
    logits = router_logits(x_bits, Wr, bias)
    x = (x_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for t in range(3):
        for e in range(5):
            exact = math.fsum([*(x[t] * Wr[e].astype(np.float64)), float(bias[e])])
            assert float(logits[t, e]) == float(np.float32(exact))
