"""LYNX AffinityBinning: confidence bins, exponentially weighted expert scores, critical set and
the remap of low-affinity tokens (oracle; test infrastructure only).

Source: LYNX, 2.1 (router confidence, from the gap between the top-ranked experts' logits,
identifies the critical token-expert mappings; the rank-0 expert dominates) and 2.2 (the
Confidence Analyzer bins each token's confidence with AffinityBinning, bin width and count set
only by the sparsity ratio k/N; the Adaptive Expert Scorer gives every expert a batch-wide score
with exponential weights of the bins, so experts preferred by high-conviction tokens score
disproportionately higher, and picks the critical set; the Expert Remapper redirects
low-affinity assignments to it, every token keeping exactly k experts).

The pages give no formula.  Reading (parity unpinned against the pages; pinned below against
closed forms, hand cases and the batch remap it reduces to):
  * confidence of token t: the fp32 gap d_t = l_(0) - l_(1) between its two largest logits
    (ranking: logit descending, lower index first on ties; d_t = 0 when E = 1 is impossible
    since k <= E and E >= 2 for a gap, so E = 1 gives d_t = +inf);
  * bins: B = ceil(N / k), width w = ln(N / k) / B (N / k <= 1: B = 1, w = +inf), and
    b_t = min(floor(d_t / w), B - 1) in float64;
  * weight 2^b_t; S_e = sum over assignments (t, s) routed to e of 2^b_t * g_ts, float64 in
    ascending (token, slot) order;
  * critical set C: every rank-0 expert, then experts outside it by S_e descending (ties ->
    lower index) until |C| = critical_n;
  * a token is low-affinity when b_t < low (default ceil(B / 2)); its slots of rank > 0 whose
    expert is not in C take, in rank order, the highest-logit expert of C not in its current set
    (ties -> lower index), keeping their gate; no candidate left -> kept.  Tokens with
    b_t >= low keep their experts.
With w = +inf every token sits in bin 0, every weight is 1 and every token is low-affinity: the
result is the batch remap of oracle.policy.remap.
"""
from __future__ import annotations

import math

import numpy as np


def default_bins(E: int, k: int):
    """(B, w, low) from the sparsity ratio k/N alone."""
    ratio = E / k
    if ratio <= 1.0:
        return 1, math.inf, 1
    B = math.ceil(ratio)
    return B, math.log(ratio) / B, (B + 1) // 2


def top2_gap(row) -> float:
    """fp32 gap between the largest and second largest logit of a row (+inf for one expert)."""
    row = np.asarray(row, dtype=np.float32)
    order = sorted(range(len(row)), key=lambda e: (-float(row[e]), e))
    if len(order) < 2:
        return math.inf
    return float(np.float32(row[order[0]]) - np.float32(row[order[1]]))


def confidence_bins(logits, B: int, w: float) -> np.ndarray:
    logits = np.asarray(logits, dtype=np.float32)
    bins = np.zeros(logits.shape[0], dtype=np.int32)
    for t in range(logits.shape[0]):
        d = top2_gap(logits[t])
        if math.isinf(w):
            b = 0
        elif math.isinf(d):
            b = B - 1
        else:
            b = min(int(math.floor(d / w)), B - 1)
        bins[t] = b
    return bins


def affinity_scores(idx, gate, bins, E: int) -> np.ndarray:
    S = [0.0] * E
    T, k = idx.shape
    for t in range(T):
        wt = 2.0 ** int(bins[t])
        for s in range(k):
            S[int(idx[t, s])] += wt * float(gate[t, s])
    return np.array(S, dtype=np.float64)


def critical_from_scores(idx, S, critical_n: int) -> np.ndarray:
    E = len(S)
    crit = np.zeros(E, dtype=np.uint8)
    for e in idx[:, 0]:
        crit[int(e)] = 1
    rest = [e for e in range(E) if not crit[e]]
    rest.sort(key=lambda e: (-S[e], e))
    for e in rest[:max(critical_n - int(crit.sum()), 0)]:
        crit[e] = 1
    return crit


def _best_in(row, allowed, current):
    best = -1
    for e in range(len(row)):
        if allowed[e] and e not in current and (best < 0 or row[e] > row[best]):
            best = e
    return best


def affinity_remap(logits, idx, gate, critical_n: int, B: int, w: float, low: int):
    """-> (idx' int32 [T,k], crit uint8 [E], bins int32 [T], scores float64 [E])."""
    logits = np.asarray(logits, dtype=np.float32)
    idx0 = np.asarray(idx, dtype=np.int32)
    gate = np.asarray(gate, dtype=np.float32)
    T, k = idx0.shape
    E = logits.shape[1]
    bins = confidence_bins(logits, B, w)
    S = affinity_scores(idx0, gate, bins, E)
    crit = critical_from_scores(idx0, S, critical_n)
    out = idx0.copy()
    for t in range(T):
        if bins[t] >= low:
            continue
        for s in range(1, k):
            if crit[int(out[t, s])]:
                continue
            cand = _best_in(logits[t], crit.astype(bool), set(int(v) for v in out[t]))
            if cand >= 0:
                out[t, s] = cand
    return out, crit, bins, S
