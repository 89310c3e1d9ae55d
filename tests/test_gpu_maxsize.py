"""Maximum sizes.  The largest batch the forward takes: T = PW_MAX_TOKENS tokens of the tiny
layer at top-2, i.e. T * k = 8192 assignments, the grouping's limit.  Both FFN paths (the tensor-core GEMM chosen by
default at 1024 tokens per expert, and the CUDA-core GEMV forced), the grouping read back from
the workspace bit-exact against the oracle's, and the whole [T, H] output against the float64
oracle.  One assignment more is refused on the host.  And the largest expert count
(PW_MAX_EXPERTS, most experts idle), the largest top-k (PW_MAX_TOPK) and k = E, routing and
grouping bit-exact, the whole output against the oracle."""
import numpy as np
import pytest

from any_precision_expert_pw_b200 import binding as B
from any_precision_expert_pw_b200.inputs import CONFIGS, make_layer
from gpu_helpers import assert_ffn_close
from oracle import layer as olayer
from test_gpu_fullsize import sampled_rows, workspace_grouping

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("tc_min", [None, 1 << 20])
def test_max_batch_both_paths(libpw, tc_min):
    import dataclasses
    from any_precision_expert_pw_b200.device_layer import DeviceLayer
    from any_precision_expert_pw_b200.inputs import POLICY_NONE
    from oracle.group import group_by_expert
    cfg = dataclasses.replace(CONFIGS["tiny"], policy=POLICY_NONE, resident_frac=None)
    T = B.PW_MAX_TOKENS
    assert T * cfg.k == 8192
    L = make_layer(cfg, T)
    D = DeviceLayer(L)
    if tc_min is not None:
        B.check(B.pw_set_tc_min_tokens(tc_min))
    try:
        D.forward()
        assert D.status() == B.PW_OK
    finally:
        B.check(B.pw_set_tc_min_tokens(4))
    ref = olayer.route(L)
    idx = ref["idx"]
    assert np.array_equal(D.idx.cpu().numpy(), idx)
    counts, offsets, perm, active = group_by_expert(idx, cfg.E)
    c, o, p, a, inv = workspace_grouping(D, T, cfg.k, cfg.E)
    assert np.array_equal(c, counts) and np.array_equal(o, offsets)
    assert np.array_equal(p, perm) and np.array_equal(a, active)
    assert np.array_equal(inv[perm], np.arange(T * cfg.k))
    y_ref = sampled_rows(L, idx, ref["gate"], list(range(T)))
    r = assert_ffn_close(D.y.cpu().numpy(), y_ref, f"tiny T={T} tc_min={tc_min}")
    print(f"max batch tiny T={T} ({'forced CUDA-core' if tc_min else 'default'}): "
          f"max|err|/rms = {r:.3e}")


def test_one_assignment_past_the_limit_is_refused(libpw):
    # T * k = 4096 * 3 > 8192: refused before any launch (the pointers are never used)
    st = B.pw_moe_anyprec_forward(256, 0, 8, 256, B.PW_MAX_TOKENS, 256, 512, 3, 256, 256, 256,
                                  256, 1 << 40)
    assert st == B.PW_ERR_UNSUPPORTED


@pytest.mark.parametrize("E,k,T", [(1024, 2, 32),    # PW_MAX_EXPERTS experts, most of them idle
                                   (32, 16, 16),     # PW_MAX_TOPK slots per token
                                   (16, 16, 4)])     # k = E: every expert routed by every token
def test_max_experts_and_slots(libpw, E, k, T):
    import dataclasses
    from any_precision_expert_pw_b200.device_layer import DeviceLayer
    from oracle.group import group_by_expert
    assert E <= B.PW_MAX_EXPERTS and k <= B.PW_MAX_TOPK
    cfg = dataclasses.replace(CONFIGS["tiny"], name=f"tiny@E{E}k{k}", E=E, k=k, renorm=True)
    L = make_layer(cfg, T)
    D = DeviceLayer(L)
    D.forward()
    assert D.status() == B.PW_OK
    ref = olayer.route(L)
    idx = ref["idx"]
    assert np.array_equal(D.idx.cpu().numpy(), idx)
    counts, offsets, perm, active = group_by_expert(idx, E)
    c, o, p, a, inv = workspace_grouping(D, T, k, E)
    assert np.array_equal(c, counts) and np.array_equal(o, offsets)
    assert np.array_equal(p, perm) and np.array_equal(a, active)
    y_ref = sampled_rows(L, idx, ref["gate"], list(range(T)))
    r = assert_ffn_close(D.y.cpu().numpy(), y_ref, f"tiny E={E} k={k} T={T}")
    print(f"tiny E={E} k={k} T={T}: max|err|/rms = {r:.3e}")
