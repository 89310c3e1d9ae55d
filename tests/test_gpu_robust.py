"""Failure paths of the fused FFN launch that a healthy run never takes, made to happen on purpose
without faulting the GPU.

* More CTAs than the GPU holds at once: the down items of an expert wait (bounded) for every
  gate_up tile of that expert.  Work items are only ever owned by CTAs that are running, so the
  forward completes with PW_OK and matches the oracle whatever part of the grid is resident.
* A wait that never completes: a test hook makes every down item wait for one gate_up
  completion more than exist; with a short wait limit the kernel gives up, records
  PW_ERR_TIMEOUT in the status word and returns.  The status reads back once and clears, and
  the next forward is PW_OK and matches the oracle (the context stays usable).

Both FFN paths (CUDA-core GEMV and tensor-core GEMM) are covered."""
import numpy as np
import pytest

from any_precision_expert_pw_b200 import binding as B
from any_precision_expert_pw_b200.inputs import CONFIGS, make_layer
from gpu_helpers import SCALED, assert_ffn_close
from oracle import layer as olayer

pytestmark = pytest.mark.gpu

PATHS = {"cuda-core": 1 << 20, "tensor-core": 0}   # pw_set_tc_min_tokens value selecting each


@pytest.fixture
def layer(libpw):
    import torch
    from any_precision_expert_pw_b200.device_layer import DeviceLayer
    L = make_layer(SCALED["mixtral"], 8)
    D = DeviceLayer(L, device="cuda:0")
    ref = olayer.moe_layer(L)
    yield torch, L, D, ref
    B.check(B.pw_set_tc_min_tokens(4))
    B.check(B.pw_set_ffn_grid(0))
    B.check(B.pw_test_hold_down_items(0))
    B.check(B.pw_set_wait_limit_ns(0))


@pytest.mark.parametrize("path", list(PATHS))
def test_oversubscribed_grid_completes(layer, path):
    torch, L, D, ref = layer
    B.check(B.pw_set_tc_min_tokens(PATHS[path]))
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for ctas in (2 * sms, 3 * sms + 1):
        B.check(B.pw_set_ffn_grid(ctas))
        D.forward()
        assert D.status() == B.PW_OK, f"{path}, {ctas} CTAs"
        assert np.array_equal(D.idx.cpu().numpy(), ref["idx"])
        assert_ffn_close(D.y.cpu().numpy(), ref["y"], f"{path}, {ctas} CTAs")


@pytest.mark.parametrize("path", list(PATHS))
def test_wait_that_never_completes_times_out(layer, path):
    torch, L, D, ref = layer
    B.check(B.pw_set_tc_min_tokens(PATHS[path]))
    B.check(B.pw_set_wait_limit_ns(5_000_000))          # 5 ms
    B.check(B.pw_test_hold_down_items(1))
    D.forward()
    assert D.status() == B.PW_ERR_TIMEOUT
    assert D.status() == B.PW_OK                          # read once, then cleared
    B.check(B.pw_test_hold_down_items(0))
    B.check(B.pw_set_wait_limit_ns(0))
    D.forward()
    assert D.status() == B.PW_OK
    assert_ffn_close(D.y.cpu().numpy(), ref["y"], f"{path}, after the timeout")


def test_test_hooks_refuse_bad_values(libpw):
    assert B.pw_set_ffn_grid(-1) == B.PW_ERR_INVALID_ARG
    assert B.pw_test_hold_down_items(-1) == B.PW_ERR_INVALID_ARG
