"""Pins for the oracle's expert-cache policy across steps (CPU only): hand-derived steps,
closed forms for the special cases, invariants on random streams."""
import math

import numpy as np

from oracle import policy as op
from oracle.cache import CacheState, cache_step
from oracle.router import softmax_topk

from any_precision_expert_pw_b200.inputs import logit_stream


def _step(st, logits, idx, gate, policy=op.POLICY_THRESHOLD, thr=0.15, beta=0.5):
    return cache_step(st, np.asarray(logits, np.float32), np.asarray(idx, np.int32),
                      np.asarray(gate, np.float32), policy, thr, beta)


def test_hand_built_admission_and_lfu_eviction():
    # E = 6, k = 2, capacity 2 (experts 0, 1 resident); 0.15 rule, beta = 0.5
    st = CacheState([1, 1, 0, 0, 0, 0])
    lo = np.array([[5.0, 4.0, 3.0, 0.0, 0.0, 0.0]], np.float32)
    # step 1: token picks 0 (hit) and 3 (miss, gate 0.1 < 0.15) -> 3 substituted by the
    # highest-logit resident not chosen: expert 1; mass[3] = 0.1
    out = _step(st, lo, [[0, 3]], [[0.9, 0.1]])
    assert out[0].tolist() == [[0, 1]] and out[1].tolist() == [[0, 2]]
    assert st.mass[3] == float(np.float32(0.1)) and st.resident.tolist() == [1, 1, 0, 0, 0, 0]
    assert st.freq.tolist() == [1, 0, 0, 1, 0, 0] and out[3:] == (0, 0, 0)
    # step 2: same choice with gate 0.45 -> substituted again (0.45 >= 0.15? yes -> fetched)
    out = _step(st, lo, [[0, 3]], [[0.55, 0.45]])
    assert out[1].tolist() == [[0, 1]]                          # fetched
    # insert 3, evict the least frequently selected unused start resident: expert 1 (freq 0)
    assert st.resident.tolist() == [1, 0, 0, 1, 0, 0] and out[3:] == (1, 0, 1)
    assert st.mass[3] == 0.0                                    # reset on insertion
    # steps 3-4 (first-choice rule): expert 4 missed with gate 0.3 is substituted (by 3, the
    # highest-logit resident not chosen) twice -> mass 0.6 >= beta -> admitted at step 4
    fc = op.POLICY_FIRST_CHOICE
    out = _step(st, lo, [[0, 4]], [[0.7, 0.3]], fc)
    assert out[0].tolist() == [[0, 3]] and out[1].tolist() == [[0, 2]] and out[4] == 0
    assert st.mass[4] == float(np.float32(0.3))
    out = _step(st, lo, [[0, 4]], [[0.7, 0.3]], fc)
    assert out[4] == 1 and out[5] == 1                          # admitted 4, evicted one
    # the victim is the start resident unused after the rewrite: 4 was substituted by 3 (the
    # highest-logit resident not chosen), so 3 is used and 0 is used -> no unused resident;
    # second tier: LFU among used {0 (freq 4), 3 (freq 2)} -> 3
    assert st.resident.tolist() == [1, 0, 0, 0, 1, 0]
    assert st.mass[4] == 0.0


def test_all_resident_only_counts_selections():
    rng = np.random.default_rng(1)
    E, k, T = 16, 4, 5
    st = CacheState(np.ones(E, np.uint8))
    seen = np.zeros(E, np.int64)
    for _ in range(6):
        lo = rng.standard_normal((T, E)).astype(np.float32)
        idx, g, _ = softmax_topk(lo, k, True)
        out = _step(st, lo, idx, g)
        assert np.array_equal(out[0], idx) and not out[1].any()
        seen += np.bincount(idx.reshape(-1), minlength=E)
    assert np.array_equal(st.freq, seen) and not st.mass.any() and st.resident.all()


def test_fetch_all_never_accumulates_mass_and_infinite_beta_never_admits():
    stream = logit_stream(64, 4, 12, seed=5, topic_len=4)
    for policy, thr, beta in ((op.POLICY_FETCH_ALL, 0.15, 0.5),
                              (op.POLICY_THRESHOLD, 0.15, math.inf)):
        res = np.zeros(64, np.uint8)
        res[:16] = 1
        st = CacheState(res)
        for lo in stream:
            idx, g, _ = softmax_topk(lo, 4, True)
            out = _step(st, lo, idx, g, policy, thr, beta)
            assert out[4] == 0                                  # no background admission
            if policy == op.POLICY_FETCH_ALL:
                assert not st.mass.any() and (out[1] != op.ACTION_SUBST).all()


def test_invariants_on_streams():
    for policy in (op.POLICY_THRESHOLD, op.POLICY_FIRST_CHOICE):
        stream = logit_stream(128, 8, 30, seed=policy, topic_len=10)
        res = np.zeros(128, np.uint8)
        res[np.random.default_rng(2).choice(128, 32, replace=False)] = 1
        st = CacheState(res)
        for lo in stream:
            idx, g, _ = softmax_topk(lo, 10, True)
            before = st.copy()
            idx2, act, m, nf, na, nev = _step(st, lo, idx, g, policy, 0.15, 0.5)
            assert st.resident.sum() == 32                      # capacity kept
            assert nf + na == nev                               # every insertion evicts one
            assert (st.mass >= 0).all()
            newly = st.resident.astype(bool) & ~before.resident.astype(bool)
            assert newly.sum() == nf + na
            assert (idx2[:, 0] == idx[:, 0]).all()              # rank 0 never substituted
