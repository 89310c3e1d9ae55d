"""Damage-greedy bitwidth planner (oracle; test infrastructure only).

Source: PagedWeight, "Composants Clés" 2 (the planner chooses each block's bitwidth from its
sensitivity and the memory budget; hot experts get higher floors and damage multipliers) and
1 / 3 (the Weight Page Table holds the committed q_i; commits happen at safe boundaries).
Reading: every block starts at its ceiling qmax; while the total bytes exceed the budget, the
block whose next one-bit step adds the least damage per byte saved,
(damage[q-1] - damage[q]) / (bytes[q] - bytes[q-1]) in float64, is lowered by one bit (ties:
lower block index; a step that saves no bytes ranks last).  Written as a plain scan over the
blocks at every step.
"""
from __future__ import annotations

import math


def plan(damage, nbytes, qmin, qmax, budget):
    """-> (q list, feasible)."""
    n = len(qmin)
    q = [int(v) for v in qmax]
    total = sum(int(nbytes[i][q[i]]) for i in range(n))
    while total > budget:
        best, best_r = -1, math.inf
        for i in range(n):
            if q[i] <= qmin[i]:
                continue
            db = int(nbytes[i][q[i]]) - int(nbytes[i][q[i] - 1])
            r = (float(damage[i][q[i] - 1]) - float(damage[i][q[i]])) / db if db > 0 else math.inf
            if best < 0 or r < best_r:
                best, best_r = i, r
        if best < 0:
            return q, False
        total -= int(nbytes[best][q[best]]) - int(nbytes[best][q[best] - 1])
        q[best] -= 1
    return q, True
