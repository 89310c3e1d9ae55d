"""pw_moe_anyprec_forward_static: the forward for callers that cannot allocate device scratch
(for instance a host program that only receives device pointers from a serving engine that owns
every GPU allocation).  It must give the same layer output as pw_moe_anyprec_forward with a
caller workspace, on two calls in a row (the second call reuses the library's scratch array,
which still holds the first call's contents).  This file is collected last on purpose."""
import numpy as np
import pytest

from any_precision_expert_pw_b200 import binding as B
from any_precision_expert_pw_b200.inputs import CONFIGS, make_layer
from gpu_helpers import FFN_RTOL_RMS, ffn_err
from oracle import layer as olayer

pytestmark = pytest.mark.gpu


def test_static_scratch_matches_workspace_forward(libpw):
    import torch
    from any_precision_expert_pw_b200.device_layer import DeviceLayer

    cfg = CONFIGS["mixtral_8x7b"].scaled(H=1152, I=1408)
    L = make_layer(cfg, 8)
    D = DeviceLayer(L)
    ref = olayer.route(L)
    idx = torch.from_numpy(np.ascontiguousarray(ref["idx"], np.int32)).to(D.device)
    gate = torch.from_numpy(np.ascontiguousarray(ref["gate"], np.float32)).to(D.device)
    assert B.pw_moe_workspace_bytes(D.T, D.k, D.E, D.H, D.I) <= B.PW_STATIC_WORKSPACE_BYTES

    D.ffn(idx_ptr=idx.data_ptr(), gate_ptr=gate.data_ptr())
    y_ws = D.y.cpu().numpy().copy()
    assert D.status() == B.PW_OK

    for call in range(2):
        y = torch.full((D.T, D.H), float("nan"), dtype=torch.float32, device=D.device)
        st = B.pw_moe_anyprec_forward_static(D.pt_dev.data_ptr(), 0, D.E, D.x.data_ptr(), D.T,
                                             D.H, D.I, D.k, idx.data_ptr(), gate.data_ptr(),
                                             y.data_ptr(), D.stream)
        assert st == B.PW_OK, B.pw_status_string(st)
        assert D.status() == B.PW_OK
        err, rms = ffn_err(y.cpu().numpy(), y_ws)
        assert err <= FFN_RTOL_RMS * rms, f"call {call}: max err {err:.3e}, rms {rms:.3e}"


def test_static_scratch_rejects_oversized_shapes(libpw):
    # a shape whose scratch need exceeds the fixed array is refused before any launch
    T, k, E, H, I = 4096, 16, 64, 8192, 8192
    assert B.pw_moe_workspace_bytes(T, k, E, H, I) > B.PW_STATIC_WORKSPACE_BYTES
    st = B.pw_moe_anyprec_forward_static(256, 0, E, 256, T, H, I, k, 256, 256, 256, 0)
    assert st == B.PW_ERR_UNSUPPORTED
