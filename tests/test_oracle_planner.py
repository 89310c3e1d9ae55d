"""Pins for the oracle's damage-greedy planner, and the C planner (pw_plan_bitwidths, host
code, no GPU) against it."""
import itertools

import numpy as np
import pytest

from any_precision_expert_pw_b200 import binding as B
from any_precision_expert_pw_b200.accounting import block_bytes
from any_precision_expert_pw_b200.inputs import synthetic_damage
from oracle.planner import plan


def _bytes_table(shapes):
    t = np.zeros((len(shapes), 9), np.uint64)
    for i, (R, C) in enumerate(shapes):
        for q in range(1, 9):
            t[i, q] = block_bytes(R, C, q)
    return t


def test_budget_extremes():
    shapes = [(64, 256)] * 5
    nb = _bytes_table(shapes)
    d = synthetic_damage(5, seed=1)
    qmin, qmax = [3] * 5, [8] * 5
    assert plan(d, nb, qmin, qmax, int(nb[:, 8].sum())) == ([8] * 5, True)
    assert plan(d, nb, qmin, qmax, int(nb[:, 3].sum())) == ([3] * 5, True)
    assert plan(d, nb, qmin, qmax, int(nb[:, 3].sum()) - 1) == ([3] * 5, False)


def test_ties_go_to_the_lower_block():
    d = np.tile(np.power(4.0, -np.arange(9.0)), (3, 1))       # identical blocks
    nb = _bytes_table([(32, 128)] * 3)
    one_step = int(nb[0, 8] - nb[0, 7])
    q, ok = plan(d, nb, [3] * 3, [8] * 3, int(nb[:, 8].sum()) - one_step)
    assert ok and q == [7, 8, 8]


def test_greedy_is_optimal_for_equal_byte_steps_with_convex_damage():
    # every one-bit step saves the same bytes and damage is convex in q: marginal analysis is
    # exact for this separable problem (real blocks' steps differ by the 2^q LUT term, so
    # there the plan is the greedy one the C planner must reproduce, not a proven optimum)
    rng = np.random.default_rng(4)
    for trial in range(6):
        n = 4
        d = synthetic_damage(n, seed=trial)
        nb = np.tile(np.arange(9, dtype=np.uint64) * 1000, (n, 1))
        qmin, qmax = [3] * n, [6] * n
        budget = int(rng.integers(int(nb[:, 3].sum()), int(nb[:, 6].sum())))
        q, ok = plan(d, nb, qmin, qmax, budget)
        best = min((sum(d[i][c[i]] for i in range(n)), c)
                   for c in itertools.product(range(3, 7), repeat=n)
                   if sum(int(nb[i][c[i]]) for i in range(n)) <= budget)
        assert ok and sum(d[i][q[i]] for i in range(n)) == pytest.approx(best[0], rel=1e-12)


def test_c_planner_matches_the_oracle(libpw):
    for seed in range(5):
        rng = np.random.default_rng(seed)
        n = 200
        shapes = [(int(rng.choice([256, 512, 1024])), int(rng.choice([512, 1024, 2048])))
                  for _ in range(n)]
        nb = _bytes_table(shapes)
        d = synthetic_damage(n, seed=seed)
        qmin = rng.integers(3, 5, size=n).astype(np.uint8)
        qmax = np.full(n, 8, np.uint8)
        lo, hi = int(sum(nb[i, qmin[i]] for i in range(n))), int(nb[:, 8].sum())
        for budget in (hi, (lo + hi) // 2, lo + 12345, lo - 1):
            q_out = np.zeros(n, np.uint8)
            dd = np.ascontiguousarray(d, np.float64)
            st = B.pw_plan_bitwidths(n, dd.ctypes.data, nb.ctypes.data, qmin.ctypes.data,
                                     qmax.ctypes.data, budget, q_out.ctypes.data)
            q_ref, ok = plan(d, nb, qmin.tolist(), qmax.tolist(), budget)
            assert q_out.tolist() == q_ref
            assert st == (B.PW_OK if ok else B.PW_ERR_UNSUPPORTED)
