"""The whole decode layer, step by step (oracle; test infrastructure only).

router GEMV -> softmax top-k -> (substitution | remap | AffinityBinning remap | nothing) ->
grouped any-precision FFN ->
gate-weighted combine, as described in the module docstrings of router, policy, group and ffn.
"""
from __future__ import annotations

import numpy as np

from . import affinity
from . import policy as pol
from .ffn import moe_ffn
from .router import router_logits, softmax_topk

POLICY_REMAP = 3
POLICY_AFFINITY = 4


def route(layer):
    """Router + top-k + the layer's assignment rewrite.  Returns a dict of the decisions."""
    cfg = layer.cfg
    logits = router_logits(layer.x_bf16, layer.Wr, layer.bias)
    idx, gate, gate64 = softmax_topk(logits, cfg.k, cfg.renorm)
    res = {"logits": logits, "idx_topk": idx, "gate": gate, "gate64": gate64, "idx": idx}
    if cfg.policy in (pol.POLICY_FETCH_ALL, pol.POLICY_THRESHOLD, pol.POLICY_FIRST_CHOICE):
        idx2, action, mass, mass64 = pol.substitute(logits, idx, gate, layer.resident, cfg.policy,
                                                    cfg.threshold)
        res.update(idx=idx2, action=action, mass=mass, mass64=mass64)
    elif cfg.policy == POLICY_REMAP:
        idx2, crit = pol.remap(logits, idx, gate, cfg.critical_n)
        res.update(idx=idx2, critical=crit)
    elif cfg.policy == POLICY_AFFINITY:
        nb, w, low = affinity.default_bins(cfg.E, cfg.k)
        idx2, crit, bins, _ = affinity.affinity_remap(logits, idx, gate, cfg.critical_n, nb, w,
                                                      low)
        res.update(idx=idx2, critical=crit, bins=bins)
    return res


def moe_layer(layer, q=None):
    """Full layer; y is float64 [T, H] (compare after rounding to fp32)."""
    res = route(layer)
    y, out = moe_ffn(layer, res["idx"], res["gate"], q=q)
    res.update(y=y, expert_out=out)
    return res

