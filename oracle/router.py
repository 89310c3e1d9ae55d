"""Router GEMV and softmax top-k (oracle; test infrastructure only).

LYNX, 1 "Énoncé du Problème": each token of the batch independently selects its k best
experts from the router output.  Readings:

* logits = x . W_r^T + bias, with x given as bf16, W_r and bias as fp32; the value is the
  float64 dot product plus bias, rounded once to fp32 (the kernel's output type).  Every
  bf16 x fp32 product is exact in float64.
* selection is taken on those fp32 logits: the k largest in descending order, equal logits
  ordered by the lower expert index.
* p = softmax over all E experts in float64; gate = p of the chosen experts, or p / sum(p of
  the chosen) when the layer renormalises; gates are rounded once to fp32.
"""
from __future__ import annotations

import numpy as np


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(
        np.float64)


def router_logits(x_bf16: np.ndarray, Wr: np.ndarray, bias: np.ndarray | None) -> np.ndarray:
    """fp32 [T, E] = round_fp32(float64(x) @ float64(W_r)^T + bias)."""
    x = bf16_bits_to_f64(x_bf16)
    acc = x @ np.asarray(Wr, dtype=np.float64).T
    if bias is not None:
        acc = acc + np.asarray(bias, dtype=np.float64)[None, :]
    return acc.astype(np.float32)


def rank_experts(logits_row: np.ndarray) -> list:
    """All experts by (logit descending, index ascending): brute-force sort."""
    vals = [float(v) for v in logits_row]
    return sorted(range(len(vals)), key=lambda e: (-vals[e], e))


def softmax(logits_row: np.ndarray) -> np.ndarray:
    l = np.asarray(logits_row, dtype=np.float64)
    z = np.exp(l - l.max())
    return z / z.sum()


def softmax_topk(logits: np.ndarray, k: int, renorm: bool):
    """-> (idx int32 [T, k], gate fp32 [T, k], gate64 float64 [T, k])."""
    logits = np.asarray(logits, dtype=np.float32)
    T, E = logits.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    idx = np.zeros((T, k), dtype=np.int32)
    gate64 = np.zeros((T, k), dtype=np.float64)
    for t in range(T):
        order = rank_experts(logits[t])[:k]
        p = softmax(logits[t])
        g = p[order]
        if renorm:
            g = g / g.sum()
        idx[t] = order
        gate64[t] = g
    return idx, gate64.astype(np.float32), gate64
