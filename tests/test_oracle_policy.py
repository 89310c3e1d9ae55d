"""Pins for the oracle's substitution, remap and grouping (CPU only)."""
import numpy as np
import pytest

from oracle.group import group_by_expert
from oracle.policy import (ACTION_FETCH, ACTION_HIT, ACTION_SUBST, POLICY_FETCH_ALL,
                           POLICY_FIRST_CHOICE, POLICY_THRESHOLD, critical_set, remap,
                           substitute)
from oracle.router import softmax_topk


def _routed(T, E, k, seed, renorm=True):
    rng = np.random.default_rng(seed)
    logits = rng.normal(0, 1.5, size=(T, E)).astype(np.float32)
    idx, gate, _ = softmax_topk(logits, k, renorm)
    return logits, idx, gate


def test_hand_built_substitution(golden):
    g = golden("substitute_e6k3.json")
    logits = np.array(g["logits"], np.float32)
    idx = np.array(g["idx"], np.int32)
    gate = np.array(g["gate"], np.float32)
    res = np.array(g["resident"], np.uint8)
    assert softmax_topk(logits, g["k"], True)[0].tolist() == g["idx"]
    for key, pol, thr in (("threshold_rule", POLICY_THRESHOLD, g["threshold"]),
                          ("first_choice", POLICY_FIRST_CHOICE, g["threshold"]),
                          ("fetch_all", POLICY_FETCH_ALL, g["threshold"])):
        i2, act, m, m64 = substitute(logits, idx, gate, res, pol, thr)
        assert i2.tolist() == g[key]["idx"], key
        assert act.tolist() == g[key]["action"], key
        assert np.allclose(m64, g[key]["mass"], rtol=0, atol=1e-7), key


@pytest.mark.parametrize("seed", range(5))
def test_substitution_invariants(seed):
    T, E, k = 16, 64, 10
    logits, idx, gate = _routed(T, E, k, seed)
    rng = np.random.default_rng(100 + seed)
    res = np.zeros(E, np.uint8)
    res[rng.choice(E, 16, replace=False)] = 1
    i2, act, m, m64 = substitute(logits, idx, gate, res, POLICY_THRESHOLD, 0.15)
    for t in range(T):
        assert len(set(i2[t].tolist())) == k                         # no duplicates
        assert act[t, 0] != ACTION_SUBST and i2[t, 0] == idx[t, 0]  # top-1 never substituted
        sub = 0.0
        for s in range(k):
            if act[t, s] == ACTION_SUBST:
                assert res[idx[t, s]] == 0 and gate[t, s] < np.float32(0.15) and s > 0
                assert res[i2[t, s]] == 1 and i2[t, s] not in idx[t]
                sub += float(gate[t, s])
            else:
                assert i2[t, s] == idx[t, s]
                assert act[t, s] == (ACTION_HIT if res[idx[t, s]] else ACTION_FETCH)
        assert m64[t] == pytest.approx(sub / float(gate[t].astype(np.float64).sum()), abs=1e-15)


def test_substitution_special_cases():
    T, E, k = 8, 32, 6
    logits, idx, gate = _routed(T, E, k, 7)
    allres = np.ones(E, np.uint8)
    i2, act, m, _ = substitute(logits, idx, gate, allres, POLICY_THRESHOLD, 0.15)
    assert np.array_equal(i2, idx) and (act == ACTION_HIT).all() and (m == 0).all()
    res = np.zeros(E, np.uint8)
    res[::3] = 1
    a = substitute(logits, idx, gate, res, POLICY_THRESHOLD, np.inf)
    b = substitute(logits, idx, gate, res, POLICY_FIRST_CHOICE, 0.15)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    c = substitute(logits, idx, gate, res, POLICY_THRESHOLD, 0.0)
    d = substitute(logits, idx, gate, res, POLICY_FETCH_ALL, 0.15)
    assert np.array_equal(c[0], idx) and np.array_equal(c[1], d[1]) and (c[2] == 0).all()


def test_hand_built_remap(golden):
    g = golden("remap_2tok.json")
    logits = np.array(g["logits"], np.float32)
    idx = np.array(g["idx"], np.int32)
    gate = np.array(g["gate"], np.float32)
    assert softmax_topk(logits, g["k"], False)[0].tolist() == g["idx"]
    i2, crit = remap(logits, idx, gate, g["critical_n"])
    assert crit.tolist() == g["critical"]
    assert i2.tolist() == g["idx_remapped"]


@pytest.mark.parametrize("T", [8, 32, 64])
def test_remap_invariants(T):
    E, k = 64, 8
    logits, idx, gate = _routed(T, E, k, T, renorm=False)
    i2, crit = remap(logits, idx, gate, 32)
    r0 = set(idx[:, 0].tolist())
    assert all(crit[e] for e in r0)
    assert int(crit.sum()) == max(32, len(r0))
    assert np.array_equal(i2[:, 0], idx[:, 0])                       # rank 0 never changed
    for t in range(T):
        assert len(set(i2[t].tolist())) == k                          # exactly k experts
        for s in range(1, k):
            assert crit[i2[t, s]] or i2[t, s] == idx[t, s]
            if i2[t, s] != idx[t, s]:
                assert not crit[idx[t, s]]
    assert len(set(i2.reshape(-1).tolist())) <= int(crit.sum())


def test_remap_special_cases():
    T, E, k = 8, 16, 4
    logits, idx, gate = _routed(T, E, k, 11, renorm=False)
    i2, crit = remap(logits, idx, gate, E)                           # C = every expert
    assert crit.all() and np.array_equal(i2, idx)
    # fewer experts carry gate mass than critical_n: zero-sum experts fill by index
    idx1 = np.array([[3, 5]], np.int32)
    gate1 = np.array([[0.6, 0.4]], np.float32)
    crit = critical_set(idx1, gate1, 8, 4)
    assert crit.tolist() == [1, 1, 0, 1, 0, 1, 0, 0]


def test_hand_built_grouping():
    counts, offsets, perm, active = group_by_expert(np.array([[1, 0], [1, 2]]), 4)
    assert counts.tolist() == [1, 2, 1, 0]
    assert offsets.tolist() == [0, 1, 3, 4, 4]
    assert perm.tolist() == [1, 0, 2, 3]
    assert active.tolist() == [0, 1, 2]


def test_grouping_is_a_stable_permutation():
    rng = np.random.default_rng(5)
    idx = rng.integers(0, 13, size=(40, 3))
    counts, offsets, perm, active = group_by_expert(idx, 13)
    assert sorted(perm.tolist()) == list(range(120))
    flat = idx.reshape(-1)
    for e in range(13):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert (flat[seg] == e).all() and (np.diff(seg) > 0).all()
