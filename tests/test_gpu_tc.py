"""Parity of the tensor-core FFN path (tcgen05 GEMM over decoded weights, fp16 operands, fp32
accumulation) against the CPU oracle, through the C ABI.  The path is forced with
pw_set_tc_min_tokens(0); the bar is the FFN bar, max |err| <= 2e-3 * rms(y).  Cases: padded
passes (batches that are not multiples of 16 tokens per expert), several passes of 64 tokens
per expert, every bitwidth 3..8, ragged ends (H or I not a multiple of the 512-column stage or
the 256-column chunk), k-sliced down projection, experts without tokens, a non-resident block,
and the plain path on the same input.
"""
import numpy as np
import pytest

from any_precision_expert_pw_b200 import binding as B
from any_precision_expert_pw_b200.inputs import CONFIGS, MOD_DOWN, make_layer
from gpu_helpers import SCALED, assert_ffn_close
from oracle import ffn as offn
from oracle import layer as olayer

pytestmark = pytest.mark.gpu

DEFAULT_MIN_TOKENS = 4


@pytest.fixture
def tc(libpw):
    import torch
    B.check(B.pw_set_tc_min_tokens(0))
    yield torch, torch.device("cuda:0")
    B.check(B.pw_set_tc_min_tokens(DEFAULT_MIN_TOKENS))


def _device_layer(L):
    from any_precision_expert_pw_b200.device_layer import DeviceLayer
    return DeviceLayer(L)


def _ffn_with(torch, D, idx, gate):
    i_d = torch.from_numpy(np.ascontiguousarray(idx, np.int32)).to(D.device)
    g_d = torch.from_numpy(np.ascontiguousarray(gate, np.float32)).to(D.device)
    D.ffn(idx_ptr=i_d.data_ptr(), gate_ptr=g_d.data_ptr())
    y = D.y.cpu().numpy()
    assert D.status() == B.PW_OK
    return y


@pytest.mark.parametrize("name,T", [("tiny", 1), ("tiny", 4), ("tiny", 64), ("tiny", 200),
                                    ("qwen15", 32), ("mixtral", 8), ("mixtral", 96),
                                    ("qwen3next", 16), ("qwen2", 32)])
def test_tc_ffn_scaled(tc, name, T):
    torch, dev = tc
    L = make_layer(SCALED[name], T)
    D = _device_layer(L)
    ref = olayer.route(L)
    y = _ffn_with(torch, D, ref["idx"], ref["gate"])
    yo, _ = offn.moe_ffn(L, ref["idx"], ref["gate"])
    assert_ffn_close(y, yo, f"{name} T={T}")


@pytest.mark.parametrize("q", [3, 4, 5, 6, 7, 8])
def test_tc_every_bitwidth(tc, q):
    torch, dev = tc
    cfg = SCALED["mixtral"]
    L = make_layer(cfg, 24)
    D = _device_layer(L)
    D.commit(list(range(2 * cfg.E)), [q] * (2 * cfg.E))
    ref = olayer.route(L)
    y = _ffn_with(torch, D, ref["idx"], ref["gate"])
    yo, _ = offn.moe_ffn(L, ref["idx"], ref["gate"], q=np.full((cfg.E, 2), q, np.uint8))
    assert_ffn_close(y, yo, f"q={q}")


def test_tc_many_passes_and_empty_experts(tc):
    torch, dev = tc
    cfg = SCALED["qwen15"]
    T = 150                                       # 150 tokens on 4 experts: passes 64, 64, 22
    L = make_layer(cfg, T)
    D = _device_layer(L)
    idx = np.array([[5, 7, 0, 59]] * T, np.int32)
    gate = np.tile(np.array([[0.4, 0.3, 0.2, 0.1]], np.float32), (T, 1))
    y = _ffn_with(torch, D, idx, gate)
    yo, _ = offn.moe_ffn(L, idx, gate)
    assert_ffn_close(y, yo, "3 passes per expert")


def test_tc_k_sliced_down(tc):
    # I = 4096 (four stages) and few down blocks: the down projection is split along k
    torch, dev = tc
    cfg = CONFIGS["tiny"].scaled(H=256, I=4096)
    L = make_layer(cfg, 32)
    D = _device_layer(L)
    ref = olayer.route(L)
    y = _ffn_with(torch, D, ref["idx"], ref["gate"])
    yo, _ = offn.moe_ffn(L, ref["idx"], ref["gate"])
    assert_ffn_close(y, yo, "k-sliced down")


def test_tc_matches_plain_path(tc):
    torch, dev = tc
    cfg = SCALED["mixtral"]
    L = make_layer(cfg, 40)
    D = _device_layer(L)
    ref = olayer.route(L)
    y_tc = _ffn_with(torch, D, ref["idx"], ref["gate"])
    B.check(B.pw_set_tc_min_tokens(1 << 30))
    y_plain = _ffn_with(torch, D, ref["idx"], ref["gate"])
    yo, _ = offn.moe_ffn(L, ref["idx"], ref["gate"])
    assert_ffn_close(y_tc, yo, "tensor-core path")
    assert_ffn_close(y_plain, yo, "plain path")
    assert_ffn_close(y_tc, y_plain, "paths against each other")


def test_tc_non_resident_block_reports_and_zeroes(tc):
    torch, dev = tc
    cfg = CONFIGS["tiny"]
    L = make_layer(cfg, 40)
    D = _device_layer(L)
    idx = np.array([[1, 2]] * 40, np.int32)
    gate = np.array([[0.5, 0.5]] * 40, np.float32)
    D.set_state(2, MOD_DOWN, B.PW_PAGE_CPU)
    i_d = torch.from_numpy(idx).to(dev)
    g_d = torch.from_numpy(gate).to(dev)
    D.ffn(idx_ptr=i_d.data_ptr(), gate_ptr=g_d.data_ptr())
    assert D.status() == B.PW_ERR_NOT_RESIDENT
    y = D.y.cpu().numpy()
    _, out = offn.moe_ffn(L, idx, gate)
    y1 = 0.5 * out[np.arange(40) * 2]                    # expert 2's contribution is zero
    assert_ffn_close(y, y1, "expert 2 skipped")
    assert D.status() == B.PW_OK


def test_tc_threshold_rejects_negative(libpw):
    assert B.pw_set_tc_min_tokens(-1) == B.PW_ERR_INVALID_ARG
