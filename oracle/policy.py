"""Residency-aware substitution and batch-aware remap (oracle; test infrastructure only).

Substitution follows "Which Expert Misses Are Worth Waiting For?", "Méthodologie": a missing
(non-resident) expert is fetched when it is the router's first choice or its gate is >= 0.15
(the 0.15 rule); the first-choice rule fetches only a missing first choice; the fetch-every-miss
baseline fetches all.  The substituted gate mass m is the normalised weighted sum of the gates
of the substituted experts.  Readings: slots are visited in rank order; a substituted slot takes
the highest-logit resident expert not in the token's current set (ties -> lower index) and keeps
its gate; m_t = (sum of substituted gates) / (sum of all the token's gates), in float64; when no
resident candidate is left the miss is fetched.

Remap follows LYNX, 2.1 (the rank-0 expert dominates quality) and 2.2 (a batch-wide score per
expert selects a minimal critical set; low-affinity assignments are redirected to it and every
token keeps exactly k experts).  Reading for this layer: S_e = sum of the gates routed to e over
the batch, a float64 sum in ascending (token, slot) order; C = every rank-0 expert, then experts
outside that set by S_e descending (ties -> lower index) until |C| = critical_n (never removing a
rank-0 expert); each slot of rank > 0 whose expert is not in C takes, in rank order, the
highest-logit expert of C not in the token's current set (ties -> lower index), keeping its
gate; with no candidate left the slot is kept.
"""
from __future__ import annotations

import numpy as np

ACTION_HIT = 0
ACTION_FETCH = 1
ACTION_SUBST = 2

POLICY_FETCH_ALL = 0
POLICY_THRESHOLD = 1
POLICY_FIRST_CHOICE = 2


def _best_candidate(logits_row, allowed, current):
    best = -1
    for e in range(len(logits_row)):
        if not allowed[e] or e in current:
            continue
        if best < 0 or logits_row[e] > logits_row[best]:
            best = e      # strict '>' in ascending index order keeps the lower index on ties
    return best


def substitute(logits, idx, gate, resident, policy: int, threshold: float):
    """-> (idx' int32 [T,k], action uint8 [T,k], mass fp32 [T], mass64 float64 [T])."""
    logits = np.asarray(logits, dtype=np.float32)
    idx = np.array(idx, dtype=np.int32, copy=True)
    gate = np.asarray(gate, dtype=np.float32)
    resident = np.asarray(resident).astype(bool)
    T, k = idx.shape
    thr = np.float32(threshold)
    action = np.zeros((T, k), dtype=np.uint8)
    mass64 = np.zeros(T, dtype=np.float64)
    for t in range(T):
        sub_sum = 0.0
        tot = 0.0
        for s in range(k):
            e = int(idx[t, s])
            g = gate[t, s]
            tot += float(g)
            if resident[e]:
                action[t, s] = ACTION_HIT
                continue
            if policy == POLICY_FETCH_ALL:
                fetch = True
            elif policy == POLICY_FIRST_CHOICE:
                fetch = (s == 0)
            elif policy == POLICY_THRESHOLD:
                fetch = (s == 0) or (g >= thr)
            else:
                raise ValueError("unknown policy")
            if not fetch:
                cand = _best_candidate(logits[t], resident, set(int(v) for v in idx[t]))
                if cand < 0:
                    fetch = True
                else:
                    idx[t, s] = cand
                    action[t, s] = ACTION_SUBST
                    sub_sum += float(g)
            if fetch:
                action[t, s] = ACTION_FETCH
        mass64[t] = sub_sum / tot if tot > 0 else 0.0
    return idx, action, mass64.astype(np.float32), mass64


def batch_gate_sum(idx, gate, E: int) -> np.ndarray:
    """S_e in float64, accumulated in ascending (token, slot) order."""
    S = [0.0] * E
    T, k = idx.shape
    for t in range(T):
        for s in range(k):
            S[int(idx[t, s])] += float(gate[t, s])
    return np.array(S, dtype=np.float64)


def critical_set(idx, gate, E: int, critical_n: int) -> np.ndarray:
    """uint8 [E] mask of the critical experts."""
    S = batch_gate_sum(idx, gate, E)
    crit = np.zeros(E, dtype=np.uint8)
    for e in idx[:, 0]:
        crit[int(e)] = 1
    rest = [e for e in range(E) if not crit[e]]
    rest.sort(key=lambda e: (-S[e], e))
    need = max(critical_n - int(crit.sum()), 0)
    for e in rest[:need]:
        crit[e] = 1
    return crit


def remap(logits, idx, gate, critical_n: int):
    """-> (idx' int32 [T,k], crit uint8 [E])."""
    logits = np.asarray(logits, dtype=np.float32)
    idx0 = np.asarray(idx, dtype=np.int32)
    gate = np.asarray(gate, dtype=np.float32)
    T, k = idx0.shape
    E = logits.shape[1]
    crit = critical_set(idx0, gate, E, critical_n)
    out = idx0.copy()
    for t in range(T):
        for s in range(1, k):
            if crit[int(out[t, s])]:
                continue
            cand = _best_candidate(logits[t], crit.astype(bool), set(int(v) for v in out[t]))
            if cand >= 0:
                out[t, s] = cand
    return out, crit
