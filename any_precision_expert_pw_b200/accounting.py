"""Algorithmic byte counts of one decode-layer call (what the method must move, no more).

Per distinct expert used after the assignment rewrite and per module: the top-q bit-planes
(R * C * q / 8 bytes) and the q-bit LUT (R * 2^q fp16 entries); plus the router weights
(E * H fp32) and bias, the activations x (T * H bf16) and the output y (T * H fp32).
"""
from __future__ import annotations

from typing import Iterable

import numpy as np


def block_bytes(R: int, C: int, q: int) -> int:
    return R * C * q // 8 + R * (1 << q) * 2


def ffn_bytes(H: int, I: int, q: np.ndarray, used: Iterable[int], T: int) -> int:
    total = 0
    for e in sorted(set(int(v) for v in used)):
        total += block_bytes(2 * I, H, int(q[e, 0])) + block_bytes(H, I, int(q[e, 1]))
    return total + T * H * 2 + T * H * 4


def layer_bytes(H: int, I: int, E: int, q: np.ndarray, used: Iterable[int], T: int,
                has_bias: bool) -> int:
    return ffn_bytes(H, I, q, used, T) + E * H * 4 + (E * 4 if has_bias else 0)


def plane_bytes(H: int, I: int, q: np.ndarray, used: Iterable[int]) -> int:
    return sum(2 * I * H * int(q[e, 0]) // 8 + H * I * int(q[e, 1]) // 8
               for e in sorted(set(int(v) for v in used)))
