"""Expert cache policy across decode steps: substitution + frequency-based eviction + background
admission (oracle; test infrastructure only).

Source: "Which Expert Misses Are Worth Waiting For?", "Méthodologie" (the 0.15 and first-choice
rules; background admission accumulates the gate weight of substituted experts over time and
admits an expert into the cache once a threshold, e.g. 0.5, is reached) and "Contributions
Clés" 5 (Quality-First = 0.15 rule + frequency-based eviction + background admission with
beta = 0.5; Speed-First = first-choice rule + frequency-based eviction + background admission).

Reading of one step (the pages give the components, not their order or tie rules):
  1. every routed assignment counts one selection of its expert: freq[e] += 1;
  2. the step's assignments are rewritten by oracle.policy.substitute against the resident set
     as it is at the start of the step (the rule does not see the step's own fetches);
  3. every substituted slot adds its gate to the missing expert it replaced:
     mass[e] += g, float64, ascending (token, slot) order;
  4. insertions: the experts fetched this step (actions FETCH on a non-resident expert), then
     every other non-resident expert with mass[e] >= beta (background admission); an inserted
     expert's mass is reset to 0;
  5. evictions keep the cache at its capacity (the number of resident experts at the start):
     victims are taken from the experts resident at the start of the step that no assignment of
     this step uses after the rewrite, least frequently selected first (ties: lower index);
     if those run out, from the remaining start-of-step residents in the same order; if the
     insertions alone exceed the capacity, the admitted experts with the least mass are dropped
     first, then fetched ones, least frequently selected first (ties: higher index dropped).
Outputs per step: the rewritten idx, actions and substituted mass m_t (as
oracle.policy.substitute), and the numbers of fetched, admitted and evicted experts.
"""
from __future__ import annotations

import numpy as np

from . import policy as pol


class CacheState:
    def __init__(self, resident):
        self.resident = np.asarray(resident, dtype=np.uint8).copy()
        E = len(self.resident)
        self.mass = np.zeros(E, dtype=np.float64)
        self.freq = np.zeros(E, dtype=np.int64)
        self.capacity = int(self.resident.sum())

    def copy(self):
        c = CacheState(self.resident)
        c.mass = self.mass.copy()
        c.freq = self.freq.copy()
        c.capacity = self.capacity
        return c


def cache_step(state: CacheState, logits, idx, gate, policy: int, threshold: float,
               beta: float):
    """Advance `state` by one step; -> (idx', action, mass32, n_fetched, n_admitted, n_evicted)."""
    idx = np.asarray(idx, dtype=np.int32)
    gate = np.asarray(gate, dtype=np.float32)
    T, k = idx.shape
    E = len(state.resident)
    start = state.resident.astype(bool).copy()
    for t in range(T):                                          # 1
        for s in range(k):
            state.freq[int(idx[t, s])] += 1
    idx2, action, mass32, _ = pol.substitute(logits, idx, gate, start, policy, threshold)  # 2
    for t in range(T):                                          # 3
        for s in range(k):
            if action[t, s] == pol.ACTION_SUBST:
                state.mass[int(idx[t, s])] += float(gate[t, s])
    fetched = []                                                # 4
    for t in range(T):
        for s in range(k):
            e = int(idx2[t, s])
            if action[t, s] == pol.ACTION_FETCH and not start[e] and e not in fetched:
                fetched.append(e)
    admitted = [e for e in range(E)
                if not start[e] and e not in fetched and state.mass[e] >= beta]
    cap = state.capacity
    if len(fetched) + len(admitted) > cap:                       # keep the best insertions
        admitted.sort(key=lambda e: (-state.mass[e], e))
        fetched.sort(key=lambda e: (-state.freq[e], e))
        keep_f = fetched[:cap]
        keep_a = admitted[:max(cap - len(keep_f), 0)]
        fetched, admitted = keep_f, keep_a
    inserted = fetched + admitted
    for e in inserted:
        state.mass[e] = 0.0
    used = set(int(v) for v in idx2.reshape(-1))
    n_over = int(start.sum()) + len(inserted) - cap             # 5
    victims = []
    if n_over > 0:
        first = sorted([e for e in range(E) if start[e] and e not in used],
                       key=lambda e: (state.freq[e], e))
        second = sorted([e for e in range(E) if start[e] and e in used],
                        key=lambda e: (state.freq[e], e))
        victims = (first + second)[:n_over]
    res = start.copy()
    for e in victims:
        res[e] = False
    for e in inserted:
        res[e] = True
    state.resident = res.astype(np.uint8)
    return idx2, action, mass32, len(fetched), len(admitted), len(victims)
