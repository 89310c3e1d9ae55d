"""Full-size parity: the pages' model shapes at their batch sizes, run through the same
DeviceLayer path as bench.py (route + rewrite + forward).  Routing and the rewrite are
compared bit-exactly over the whole batch, the grouping bit-exactly against the oracle's, and
the whole [T, H] FFN output element by element against the float64 oracle (max |err| <=
2e-3 * rms(y))."""
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
    """y[t] for the given tokens (all of them: the oracle's whole layer output): each expert they
    use is evaluated once on those tokens, in float64."""
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


def workspace_grouping(D, T, k, E):
    """counts, offsets, perm and the active experts as the forward left them at the start of its
    workspace (layout in include/pw.h, pw_moe_workspace_bytes: int32 regions counts[E],
    offsets[E+1], perm[T*k], inv[T*k], active[E], meta[8], each at a 256-byte boundary)."""
    ws = D.workspace.cpu().numpy()
    up = lambda n: (n + 255) // 256 * 256
    o_counts = 0
    o_offsets = o_counts + up(4 * E)
    o_perm = o_offsets + up(4 * (E + 1))
    o_inv = o_perm + up(4 * T * k)
    o_active = o_inv + up(4 * T * k)
    o_meta = o_active + up(4 * E)
    i32 = lambda o, n: ws[o:o + 4 * n].view(np.int32)
    n_active = int(i32(o_meta, 1)[0])
    return (i32(o_counts, E), i32(o_offsets, E + 1), i32(o_perm, T * k),
            i32(o_active, n_active), i32(o_inv, T * k))


# every config at its model shape and the batch sizes of its sweep; the last two are
# prefill-sized batches (the tensor-core FFN, several 64-token passes per expert; routing by plain
# top-k, as a phase-aware schedule would do without the decode remap)
@pytest.mark.parametrize("name,T,plain", [("qwen15_moe_a2.7b", 32, False),
                                          ("qwen3_next_80b_a3b", 1, False),
                                          ("qwen3_next_80b_a3b", 16, False),
                                          ("qwen2_57b_a14b", 8, False),
                                          ("qwen2_57b_a14b", 32, False),
                                          ("qwen2_57b_a14b", 64, False),
                                          ("mixtral_8x7b", 8, False),
                                          ("mixtral_8x7b", 64, False),
                                          ("mixtral_8x7b", 256, False),
                                          ("mixtral_8x7b", 512, True),
                                          ("qwen2_57b_a14b", 512, True)])
def test_full_size_layer(torch_dev, name, T, plain):
    torch, dev = torch_dev
    import dataclasses
    from any_precision_expert_pw_b200.device_layer import DeviceLayer
    from any_precision_expert_pw_b200.inputs import POLICY_NONE
    from oracle.group import group_by_expert
    cfg = CONFIGS[name]
    if plain:
        cfg = dataclasses.replace(cfg, policy=POLICY_NONE, resident_frac=None)
    L = make_layer(cfg, T)
    D = DeviceLayer(L)
    D.forward()
    assert D.status() == B.PW_OK
    ref = olayer.route(L)
    idx = ref["idx"]
    assert np.array_equal(D.idx.cpu().numpy(), idx)
    # the grouping the FFN ran on, bit-exact
    counts, offsets, perm, active = group_by_expert(idx, cfg.E)
    c, o, p, a, inv = workspace_grouping(D, T, cfg.k, cfg.E)
    assert np.array_equal(c, counts) and np.array_equal(o, offsets)
    assert np.array_equal(p, perm) and np.array_equal(a, active)
    assert np.array_equal(inv[perm], np.arange(T * cfg.k))
    # the whole output against the oracle's layer (its own routing and gates)
    y_ref = sampled_rows(L, idx, ref["gate"], list(range(T)))
    r = assert_ffn_close(D.y.cpu().numpy(), y_ref, f"{name} T={T}")
    print(f"full-size {name} T={T}: max|err|/rms = {r:.3e}")
