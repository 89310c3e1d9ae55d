"""Pins for the oracle's any-precision FFN and combine (CPU only)."""
import math

import numpy as np
import pytest

from any_precision_expert_pw_b200.inputs import CONFIGS, f32_to_bf16_bits, make_layer
from oracle.ffn import block_matvec, dequant_rows, expert_ffn, moe_ffn, silu
from oracle.router import softmax_topk


def test_hand_built_expert(golden):
    g = golden("ffn_hand.json")
    n = g["n"]
    gu, dn = g["gate_up"], g["down"]
    X = np.array([g["x"]], np.float64)
    out = expert_ffn(np.array(gu["idx"], np.uint8), np.array(gu["lut"], np.float16), gu["q"],
                     np.array(dn["idx"], np.uint8), np.array(dn["lut"], np.float16), dn["q"],
                     n, X)
    assert out[0].tolist() == pytest.approx(g["out"], rel=1e-15)
    GU = block_matvec(np.array(gu["idx"], np.uint8), np.array(gu["lut"], np.float16), n,
                      gu["q"], X.T)
    assert GU[:, 0].tolist() == [g["gate"], g["up"]]


def test_silu_closed_forms():
    assert silu(0.0) == 0.0
    assert silu(math.log(3.0)) == pytest.approx(0.75 * math.log(3.0), rel=1e-15)
    z = np.linspace(-30, 30, 121)
    assert np.allclose(silu(z) - silu(-z), z, rtol=0, atol=1e-13)     # silu(z) - silu(-z) = z
    assert silu(40.0) == pytest.approx(40.0, rel=1e-15)
    assert abs(silu(-800.0)) == 0.0


@pytest.mark.parametrize("q", [1, 3, 4])
def test_integer_lut_exposes_decoded_index(q):
    # with lut[r][v] = v and one-hot x, W x returns the q-bit index column itself
    n = 4
    rng = np.random.default_rng(q)
    idx = rng.integers(0, 16, size=(6, 64), dtype=np.uint8)
    lut = np.tile(np.arange(1 << q, dtype=np.float16), (6, 1))
    for c in (0, 31, 32, 63):
        X = np.zeros((64, 1))
        X[c, 0] = 1.0
        col = block_matvec(idx, lut, n, q, X, row_chunk=4)[:, 0]
        assert col.tolist() == (idx[:, c] >> (n - q)).astype(float).tolist()


def test_full_bitwidth_equals_dense_lut_dequant():
    n = 8
    rng = np.random.default_rng(3)
    idx = rng.integers(0, 256, size=(5, 64), dtype=np.uint8)
    lut = rng.normal(0, 0.02, size=(5, 256)).astype(np.float16)
    W = dequant_rows(idx, lut, n, n)
    for r in range(5):
        for c in range(64):
            assert W[r, c] == float(lut[r, idx[r, c]])


def test_brute_force_loops_tiny_layer():
    # pure-Python scalar loops over a tiny two-slot layer, against the vectorised oracle
    n, H, I, E, T, k = 4, 4, 3, 3, 3, 2
    rng = np.random.default_rng(9)
    idx = [[rng.integers(0, 16, size=(2 * I, H), dtype=np.uint8),
            rng.integers(0, 16, size=(H, I), dtype=np.uint8)] for _ in range(E)]
    qs = np.array([[3, 4], [4, 3], [2, 2]], np.uint8)
    luts = [[rng.normal(0, 0.5, size=(2 * I, 1 << int(qs[e, 0]))).astype(np.float16),
             rng.normal(0, 0.5, size=(H, 1 << int(qs[e, 1]))).astype(np.float16)] for e in range(E)]
    x_bits = f32_to_bf16_bits(rng.normal(size=(T, H)).astype(np.float32))
    x = (x_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    sel = np.array([[2, 0], [1, 2], [0, 1]], np.int32)
    gate = np.array([[0.7, 0.3], [0.5, 0.5], [0.9, 0.1]], np.float32)

    class L:  # minimal layer view for moe_ffn
        pass
    lay = L()
    lay.cfg = type("C", (), {"E": E, "n": n, "H": H})()
    lay.q, lay.x_bf16 = qs, x_bits
    lay.idx = idx
    lay.lut = [[{int(qs[e, 0]): luts[e][0]}, {int(qs[e, 1]): luts[e][1]}] for e in range(E)]
    y, _ = moe_ffn(lay, sel, gate)

    def w(e, m, r, c):
        q = int(qs[e, m])
        return float(luts[e][m][r, int(idx[e][m][r, c]) >> (n - q)])

    for t in range(T):
        yt = [0.0] * H
        for s in range(k):
            e = int(sel[t, s])
            h = []
            for i in range(I):
                gsum = sum(w(e, 0, i, c) * x[t, c] for c in range(H))
                usum = sum(w(e, 0, I + i, c) * x[t, c] for c in range(H))
                h.append(gsum / (1 + math.exp(-gsum)) * usum)
            for r in range(H):
                yt[r] += float(gate[t, s]) * sum(w(e, 1, r, i) * h[i] for i in range(I))
        assert y[t].tolist() == pytest.approx(yt, rel=1e-12, abs=1e-15)


def test_combine_single_expert_and_permutation():
    cfg = CONFIGS["tiny"]
    L = make_layer(cfg, 4)
    T, k = 4, cfg.k
    sel = np.tile(np.array([[3, 5]], np.int32), (T, 1))
    one = np.tile(np.array([[1.0, 0.0]], np.float32), (T, 1))
    y, out = moe_ffn(L, sel, one)
    q = L.q
    X = (L.x_bf16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = expert_ffn(L.idx[3][0], L.lut[3][0][int(q[3, 0])], int(q[3, 0]),
                     L.idx[3][1], L.lut[3][1][int(q[3, 1])], int(q[3, 1]), cfg.n, X)
    assert np.allclose(y, ref, rtol=1e-13, atol=0)
    # permuting tokens permutes outputs
    logits = np.random.default_rng(1).normal(size=(T, cfg.E)).astype(np.float32)
    idx, gate, _ = softmax_topk(logits, k, False)
    y1, _ = moe_ffn(L, idx, gate)
    p = np.array([2, 0, 3, 1])
    L2 = make_layer(cfg, 4)
    L2.x_bf16 = L.x_bf16[p]
    y2, _ = moe_ffn(L2, idx[p], gate[p])
    assert np.allclose(y2, y1[p], rtol=1e-13, atol=0)
