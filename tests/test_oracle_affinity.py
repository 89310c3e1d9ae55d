"""Pins for the oracle's AffinityBinning reading (CPU only).  The pages give no formula, so
parity with the pages is unpinned; these pin the reading against hand-derived cases, closed
forms, brute force and the batch remap it reduces to."""
import math

import numpy as np
import pytest

from oracle import affinity as oa
from oracle import policy as op
from oracle.router import softmax_topk



def test_default_bins_follow_the_sparsity_ratio():
    assert oa.default_bins(64, 8) == (8, math.log(8.0) / 8, 4)       # Qwen2-shaped
    assert oa.default_bins(8, 2) == (4, math.log(4.0) / 4, 2)        # Mixtral-shaped
    B, w, low = oa.default_bins(512, 10)                             # ratio 51.2
    assert (B, low) == (52, 26) and w == pytest.approx(math.log(51.2) / 52)
    assert oa.default_bins(4, 4) == (1, math.inf, 1)                 # k = N: one bin


def test_hand_case_bins_scores_and_remap():
    # E = 6, k = 2, three tokens; w = 0.5, B = 4, low = 2
    logits = np.array([[3.0, 1.0, 0.5, 0.0, 0.0, 0.0],     # gap 2.0 -> bin 3 (capped)
                       [0.0, 1.2, 1.0, 0.0, 0.9, 0.0],     # gap 0.2 -> bin 0
                       [0.0, 0.0, 2.0, 1.3, 0.0, 1.0]],    # gap 0.7 -> bin 1
                      dtype=np.float32)
    idx = np.array([[0, 1], [1, 2], [2, 3]], dtype=np.int32)
    gate = np.array([[0.6, 0.4], [0.5, 0.5], [0.7, 0.3]], dtype=np.float32)
    bins = oa.confidence_bins(logits, 4, 0.5)
    assert bins.tolist() == [3, 0, 1]
    S = oa.affinity_scores(idx, gate, bins, 6)
    f = lambda v: float(np.float32(v))
    # expert 1: 8*0.4 (token 0) + 1*0.5 (token 1); expert 2: 0.5 + 2*0.7; expert 3: 2*0.3
    assert S[1] == 8 * f(0.4) + f(0.5)
    assert S[2] == f(0.5) + 2 * f(0.7)
    assert S[3] == 2 * f(0.3) and S[4] == 0.0
    # C with critical_n = 3: rank-0 experts {0, 1, 2}; nothing else fits
    out, crit, _, _ = oa.affinity_remap(logits, idx, gate, 3, 4, 0.5, 2)
    assert crit.tolist() == [1, 1, 1, 0, 0, 0]
    # token 0 (bin 3) and token 2 (bin 1 < 2 -> low) : token 2's slot 1 (expert 3, not
    # critical) -> highest-logit critical expert not chosen: logits row 2 over {0, 1} = 0, 0
    # -> expert 0 (lower index); token 1's slot 1 expert 2 is critical -> kept
    assert out.tolist() == [[0, 1], [1, 2], [2, 0]]


def test_high_conviction_token_outweighs_heavier_low_conviction_gate():
    # expert 3 gets gate 0.3 from a bin-3 token (weight 8 -> 2.4); expert 4 gets 0.9 from two
    # bin-0 tokens (0.45 each); with one free critical slot expert 3 wins
    logits = np.array([[5.0, 0, 0, 1.0, 0, 0],
                       [1.0, 0, 0, 0, 0.95, 0],
                       [0, 1.0, 0, 0, 0.95, 0]], dtype=np.float32)
    idx = np.array([[0, 3], [0, 4], [1, 4]], dtype=np.int32)
    gate = np.array([[0.7, 0.3], [0.55, 0.45], [0.55, 0.45]], dtype=np.float32)
    out, crit, bins, S = oa.affinity_remap(logits, idx, gate, 3, 4, 0.5, 2)
    assert bins.tolist() == [3, 0, 0]
    assert crit.tolist() == [1, 1, 0, 1, 0, 0]
    # without the weights (batch gate sums) expert 4 would have won the slot
    assert op.critical_set(idx, gate, 6, 3).tolist() == [1, 1, 0, 0, 1, 0]


def test_infinite_width_reduces_to_the_batch_remap():
    rng = np.random.default_rng(7)
    for _ in range(5):
        T, E, k = 16, 24, 4
        logits = rng.standard_normal((T, E)).astype(np.float32)
        idx, gate, _ = softmax_topk(logits, k, renorm=False)
        want, crit_want = op.remap(logits, idx, gate, 8)
        got, crit, bins, _ = oa.affinity_remap(logits, idx, gate, 8, 1, math.inf, 1)
        assert np.array_equal(got, want) and np.array_equal(crit, crit_want)
        assert not bins.any()


def test_no_low_bins_is_the_identity():
    rng = np.random.default_rng(3)
    logits = rng.standard_normal((10, 16)).astype(np.float32)
    idx, gate, _ = softmax_topk(logits, 4, renorm=True)
    B, w, _ = oa.default_bins(16, 4)
    out, _, _, _ = oa.affinity_remap(logits, idx, gate, 4, B, w, 0)
    assert np.array_equal(out, idx)


def test_bins_match_brute_force_definition():
    rng = np.random.default_rng(11)
    logits = (rng.standard_normal((200, 12)) * 2).astype(np.float32)
    B, w, _ = oa.default_bins(12, 3)
    bins = oa.confidence_bins(logits, B, w)
    for t in range(200):
        srt = sorted(logits[t].tolist(), reverse=True)
        d = float(np.float32(srt[0]) - np.float32(srt[1]))
        assert bins[t] == min(math.floor(d / w), B - 1)


def test_invariants_on_random_batches():
    for seed in range(4):
        T, E, k, crit_n = 32, 64, 8, 32
        rng = np.random.default_rng(seed)
        logits = (rng.standard_normal((T, E)) * 1.2).astype(np.float32)
        idx, gate, _ = softmax_topk(logits, k, renorm=False)
        B, w, low = oa.default_bins(E, k)
        out, crit, bins, _ = oa.affinity_remap(logits, idx, gate, crit_n, B, w, low)
        for t in range(T):
            assert len(set(out[t].tolist())) == k               # k distinct experts
            assert out[t, 0] == idx[t, 0]                        # rank 0 never remapped
            if bins[t] >= low:
                assert np.array_equal(out[t], idx[t])            # high affinity: untouched
            for s in range(k):
                if out[t, s] != idx[t, s]:
                    assert crit[out[t, s]]                       # remapped into C
        assert crit.sum() == max(crit_n, len(set(idx[:, 0].tolist())))
