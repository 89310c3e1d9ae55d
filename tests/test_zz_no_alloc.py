"""pw_moe_anyprec_forward_static: the forward for callers that cannot allocate device scratch
(for instance a host program that only receives device pointers from a serving engine that owns
every GPU allocation).  It must give the same layer output as pw_moe_anyprec_forward with a
caller workspace, and the oracle's, on two calls in a row (the second call reuses the library's
scratch array, which still holds the first call's contents), on both FFN paths.  This file is
collected last on purpose: if it fails, a run that stops at the first failure has already run
every other test."""
import numpy as np
import pytest

from any_precision_expert_pw_b200 import binding as B
from any_precision_expert_pw_b200.inputs import CONFIGS, make_layer
from gpu_helpers import FFN_RTOL_RMS, ffn_err
from oracle import layer as olayer

pytestmark = pytest.mark.gpu

# (shape, T, pw_set_tc_min_tokens value): the CUDA-core path (scaled Mixtral-shaped layer,
# 16 assignments over 8 experts) and the tensor-core path (forced), the Mixtral-shaped layer at
# full size and batch 16 among them (its scratch need is close to the array's size), and the
# Qwen1.5-shaped layer at batch 64 (the tensor-core path by default, several experts per CTA)
CASES = [("mixtral_scaled", 8, None), ("mixtral_scaled", 8, 0), ("mixtral_8x7b", 16, None),
         ("mixtral_8x7b", 16, 0), ("qwen15_moe_a2.7b", 64, None)]


def _cfg(name):
    if name == "mixtral_scaled":
        return CONFIGS["mixtral_8x7b"].scaled(H=1152, I=1408)
    return CONFIGS[name]


@pytest.mark.parametrize("name,T,tc_min", CASES)
def test_static_scratch_matches_workspace_forward_and_oracle(libpw, name, T, tc_min):
    import torch
    from any_precision_expert_pw_b200.device_layer import DeviceLayer

    L = make_layer(_cfg(name), T)
    D = DeviceLayer(L)
    ref = olayer.moe_layer(L)
    idx = torch.from_numpy(np.ascontiguousarray(ref["idx"], np.int32)).to(D.device)
    gate = torch.from_numpy(np.ascontiguousarray(ref["gate"], np.float32)).to(D.device)
    assert B.pw_moe_workspace_bytes(D.T, D.k, D.E, D.H, D.I) <= B.PW_STATIC_WORKSPACE_BYTES
    if tc_min is not None:
        B.check(B.pw_set_tc_min_tokens(tc_min))
    try:
        D.ffn(idx_ptr=idx.data_ptr(), gate_ptr=gate.data_ptr())
        y_ws = D.y.cpu().numpy().copy()
        assert D.status() == B.PW_OK
        for call in range(2):
            y = torch.full((D.T, D.H), float("nan"), dtype=torch.float32, device=D.device)
            st = B.pw_moe_anyprec_forward_static(D.pt_dev.data_ptr(), 0, D.E, D.x.data_ptr(),
                                                 D.T, D.H, D.I, D.k, idx.data_ptr(),
                                                 gate.data_ptr(), y.data_ptr(), D.stream)
            assert st == B.PW_OK, B.pw_status_string(st)
            assert D.status() == B.PW_OK
            got = y.cpu().numpy()
            for what, want in (("workspace forward", y_ws), ("oracle", ref["y"])):
                err, rms = ffn_err(got, want)
                assert err <= FFN_RTOL_RMS * rms, f"call {call} vs {what}: {err:.3e}, rms {rms:.3e}"
    finally:
        B.check(B.pw_set_tc_min_tokens(4))


def test_static_scratch_rejects_oversized_shapes(libpw):
    # a valid shape whose scratch need exceeds the fixed array is refused before any launch
    T, k, E, H, I = 4096, 2, 64, 8192, 8192
    assert B.pw_moe_workspace_bytes(T, k, E, H, I) > B.PW_STATIC_WORKSPACE_BYTES
    st = B.pw_moe_anyprec_forward_static(256, 0, E, 256, T, H, I, k, 256, 256, 256, 0)
    assert st == B.PW_ERR_UNSUPPORTED


def test_static_scratch_argument_errors_match_the_workspace_forward(libpw):
    # the same bad arguments give the same status from both entry points, whatever the shape's
    # scratch need: H % 128 != 0, k > E, T beyond PW_MAX_TOKENS, a null pointer
    fwd, static = B.pw_moe_anyprec_forward, B.pw_moe_anyprec_forward_static
    for T, k, E, H, I, x in [(4, 2, 8, 200, 512, 256), (4, 9, 8, 256, 512, 256),
                             (B.PW_MAX_TOKENS + 1, 2, 8, 8192, 8192, 256),
                             (4096, 2, 64, 8192, 8192, 0)]:
        want = fwd(256, 0, E, x, T, H, I, k, 256, 256, 256, 256, 1 << 40)
        assert want == B.PW_ERR_INVALID_ARG
        assert static(256, 0, E, x, T, H, I, k, 256, 256, 256, 0) == want
