"""Bit-plane packing and decoding (oracle; test infrastructure only).

PagedWeight, "Composants Clés" 1: weights are stored in a stacked bit-plane format with
look-up tables.  Reading of the layout: n planes, plane p holds bit (n-1-p) of every parent
index (plane 0 is the most significant bit), row-major per plane, 32 columns per uint32 word,
column 32w+j at bit j of word w.  A b-bit view of the block reads the top b planes; its index
is the top b bits of the parent index.
"""
from __future__ import annotations

import numpy as np


def pack_bitplanes(idx: np.ndarray, n: int) -> np.ndarray:
    """uint8 parent indices [R, C] -> uint32 planes [n, R, C/32] (naive: bit by bit)."""
    idx = np.asarray(idx, dtype=np.uint8)
    R, C = idx.shape
    if C % 32:
        raise ValueError("columns must be a multiple of 32")
    planes = np.zeros((n, R, C // 32), dtype=np.uint32)
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))      # 2^j for column j of a word
    for p in range(n):
        bit = ((idx >> (n - 1 - p)) & 1).astype(np.uint64).reshape(R, C // 32, 32)
        planes[p] = (bit * weights).sum(axis=2).astype(np.uint32)
    return planes


def unpack_bitplanes(planes: np.ndarray, q: int) -> np.ndarray:
    """Top-q planes [>=q, R, W] -> q-bit indices [R, 32W]: sum_p bit_p * 2^(q-1-p)."""
    _, R, W = planes.shape
    out = np.zeros((R, W * 32), dtype=np.int64)
    for p in range(q):
        words = planes[p].astype(np.uint64)
        for j in range(32):
            bit = (words >> np.uint64(j)) & np.uint64(1)
            out[:, j::32] += bit.astype(np.int64) << (q - 1 - p)
    return out


def child_index(idx: np.ndarray, n: int, q: int) -> np.ndarray:
    """q-bit index from the n-bit parent index: its top q bits."""
    return (np.asarray(idx).astype(np.int64) >> (n - q))
