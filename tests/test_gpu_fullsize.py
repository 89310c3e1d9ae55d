"""Full-size parity: the pages' model shapes at their batch sizes, run through the same
DeviceLayer path as bench.py (route + rewrite + forward).  Routing and the rewrite are
compared bit-exactly over the whole batch; the FFN output on a seeded sample of tokens, whose
rows the oracle computes on its own (max |err| <= 2e-3 * rms over the sampled rows)."""
import numpy as np
import pytest

from any_precision_expert_pw_b200 import binding as B
from any_precision_expert_pw_b200.inputs import CONFIGS, make_layer
from gpu_helpers import assert_ffn_close
from oracle import layer as olayer
from oracle.ffn import expert_ffn
from oracle.router import bf16_bits_to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_dev(libpw):
    import torch
    return torch, torch.device("cuda:0")


def sampled_rows(L, idx, gate, tokens):
    """y[t] for the given tokens: each expert they use is evaluated once on those tokens."""
    k = idx.shape[1]
    X = bf16_bits_to_f64(L.x_bf16)
    n = L.cfg.n
    y = np.zeros((len(tokens), L.cfg.H))
    experts = sorted({int(idx[t, s]) for t in tokens for s in range(k)})
    for e in experts:
        rows = [(i, s) for i, t in enumerate(tokens) for s in range(k) if idx[t, s] == e]
        Xe = X[[tokens[i] for i, _ in rows]]
        qg, qd = int(L.q[e, 0]), int(L.q[e, 1])
        o = expert_ffn(L.idx[e][0], L.lut[e][0][qg], qg, L.idx[e][1], L.lut[e][1][qd], qd, n, Xe)
        for j, (i, s) in enumerate(rows):
            y[i] += float(gate[tokens[i], s]) * o[j]
    return y


# the last two are prefill-sized batches (the tensor-core FFN, several 64-token passes per
# expert; routing by plain top-k, as a phase-aware schedule would do without the decode remap)
@pytest.mark.parametrize("name,T,nsample,plain", [("qwen15_moe_a2.7b", 32, 4, False),
                                                  ("qwen3_next_80b_a3b", 16, 4, False),
                                                  ("qwen2_57b_a14b", 64, 3, False),
                                                  ("mixtral_8x7b", 64, 3, False),
                                                  ("mixtral_8x7b", 256, 3, False),
                                                  ("mixtral_8x7b", 512, 2, True),
                                                  ("qwen2_57b_a14b", 512, 2, True)])
def test_full_size_layer_sampled(torch_dev, name, T, nsample, plain):
    torch, dev = torch_dev
    import dataclasses
    from any_precision_expert_pw_b200.device_layer import DeviceLayer
    from any_precision_expert_pw_b200.inputs import POLICY_NONE
    cfg = CONFIGS[name]
    if plain:
        cfg = dataclasses.replace(cfg, policy=POLICY_NONE, resident_frac=None)
    L = make_layer(cfg, T)
    D = DeviceLayer(L)
    D.forward()
    assert D.status() == B.PW_OK
    ref = olayer.route(L)
    assert np.array_equal(D.idx.cpu().numpy(), ref["idx"])
    rng = np.random.default_rng(T)
    tokens = sorted(rng.choice(T, size=nsample, replace=False).tolist())
    # y is combined with the GPU's own fp32 gates (within 1e-6 of the oracle's)
    y_ref = sampled_rows(L, ref["idx"], D.gate.cpu().numpy(), tokens)
    y = D.y.cpu().numpy()[tokens]
    assert_ffn_close(y, y_ref, f"{name} T={T} tokens {tokens}")
