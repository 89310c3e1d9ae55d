"""Token -> expert grouping (oracle; test infrastructure only).

LYNX, 1 "Énoncé du Problème": the set of experts to load grows with the batch because every
token picks its own.  The grouped layout lists, for each expert, the assignments routed to it.
Reading: assignment a = t*k + slot; within an expert the assignments are in ascending a.
"""
from __future__ import annotations

import numpy as np


def group_by_expert(idx, E: int):
    """-> (counts int32 [E], offsets int32 [E+1], perm int32 [T*k], active int32 [n_active])."""
    flat = np.asarray(idx, dtype=np.int64).reshape(-1)
    lists = [[] for _ in range(E)]
    for a, e in enumerate(flat):
        lists[int(e)].append(a)
    counts = np.array([len(l) for l in lists], dtype=np.int32)
    offsets = np.zeros(E + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    perm = np.array([a for l in lists for a in l], dtype=np.int32)
    active = np.array([e for e in range(E) if counts[e] > 0], dtype=np.int32)
    return counts, offsets, perm, active
