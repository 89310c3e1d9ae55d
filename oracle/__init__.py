"""CPU oracle for the any-precision MoE decode layer -- TEST INFRASTRUCTURE ONLY.

Plain, slow, float64 NumPy restatement of what the decode layer computes.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py`` may import it; the product path (the ``pw_*`` C library and its binding) never
does, and the oracle imports nothing from it.  The two share only the seeded input generator
(``any_precision_expert_pw_b200.inputs``), which holds none of the layer's arithmetic.

Sources (page title and section; the pages are summaries in French):

* PagedWeight, "Composants Clés" 1 -- per-(layer, expert, module) linear blocks, Any-Precision
  stacked bit-planes with look-up tables, and a Weight Page Table that holds the committed
  bitwidth q_i of each block.
* PagedWeight, "Composants Clés" 3 -- one fused mixed-precision kernel reads the bit-planes and
  LUTs directly, each block at its own bitwidth; commits happen at safe boundaries.
* "Which Expert Misses Are Worth Waiting For?", "Méthodologie" -- substituted gate mass m and the
  fetch-every-miss, 0.15 and first-choice rules.
* LYNX, 2.1 "Principes Fondamentaux" (rank-0 dominates) and 2.2 "Composants du Système"
  (batch-wide expert scores, a critical expert set, remapping that keeps exactly k experts).
* LYNX, 1 "Énoncé du Problème" -- each token independently picks its top-k experts.
* LYNX, 2.2 "Composants du Système" (Confidence Analyzer, Adaptive Expert Scorer) and 3 item 2
  -- AffinityBinning (affinity.py).

Everything the pages leave open is read the plainest way and stated where it is used: the
plane layout (plane 0 = most significant bit, bit j of word w = column 32w+j), child index =
top b bits of the parent index, gate rows before up rows in gate_up, SiLU(gate)*up, softmax over
all experts with an index tie-break, the gate compared against 0.15 being the routing gate, the
batch gate sum S_e being a float64 sum in ascending (token, slot) order, and the gate-weighted
combine in slot order.

Pins (tests/test_oracle_*.py check the oracle against things other than itself): brute force
on tiny cases, hand-built golden cases under tests/golden/, closed forms (SiLU identities,
two-expert softmax), special cases (q = n equals the dense LUT-dequantised matrix, one-hot and
integer-valued LUTs that expose the decoded indices, all-resident = identity, +inf threshold =
first-choice rule, critical set covering every chosen expert = identity), and invariants
(exactly k distinct experts per token, top-1 never substituted, rank-0 never remapped).

Parity unpinned: affinity.py (AffinityBinning).  The pages name its parts but give no formula,
so what it computes is this project's reading (stated in its docstring); it is pinned against
hand cases, a brute-force bin definition and the batch remap it reduces to, not against the
pages.  Every other function is pinned as above.
"""
from . import affinity, bitplanes, router, policy, group, ffn, layer  # noqa: F401
