"""Parity of the CUDA path (through the C ABI) against the CPU oracle.

Bit-exact: packed planes, routing indices, substitution actions, remap decisions, critical
set.  Within tolerance: logits (<= 1 ulp), gates and substituted mass (1e-6), FFN output
(max |err| <= 2e-3 * rms).  Every oracle input comes from the seeded generator."""
import numpy as np
import pytest

from any_precision_expert_pw_b200 import binding as B
from any_precision_expert_pw_b200.inputs import (CONFIGS, MOD_DOWN, MOD_GATE_UP, POLICY_REMAP,
                                                 make_layer, random_indices,
                                                 random_router_inputs)
from gpu_helpers import GATE_ATOL, SCALED, assert_ffn_close, tiled_reference
from oracle import bitplanes as obp
from oracle import ffn as offn
from oracle import layer as olayer
from oracle import policy as opol
from oracle import router as orouter

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_dev(libpw):
    import torch
    return torch, torch.device("cuda:0")


def _stream(torch):
    return torch.cuda.current_stream().cuda_stream


# ------------------------------------------------------------------ K0 pack
@pytest.mark.parametrize("rows,cols,n", [(32, 128, 4), (96, 4096, 8), (64, 1408, 8), (7, 96, 3)])
def test_pack_bit_exact(torch_dev, rows, cols, n):
    torch, dev = torch_dev
    idx = random_indices(rows, cols, n, seed=rows + cols)
    idx_d = torch.from_numpy(idx).to(dev)
    ref = obp.pack_bitplanes(idx, n)
    layouts = [B.PW_LAYOUT_ROWS]
    if rows % 32 == 0 and cols % 128 == 0:
        layouts += [B.PW_LAYOUT_TILED_GATE_UP, B.PW_LAYOUT_TILED_DOWN]
    for layout in layouts:
        planes = torch.full((n * rows * (cols // 32),), -1, dtype=torch.int32, device=dev)
        B.check(B.pw_pack_bitplanes(idx_d.data_ptr(), rows, cols, n, layout, planes.data_ptr(),
                                    _stream(torch)))
        got = planes.cpu().numpy().view(np.uint32)
        want = ref.reshape(-1) if layout == B.PW_LAYOUT_ROWS else tiled_reference(ref, layout)
        assert np.array_equal(got, want), f"layout {layout}"
    assert B.pw_get_status(_stream(torch)) == B.PW_OK


# ------------------------------------------------------------------ K1 router
def _route_gpu(torch, dev, x_bits, Wr, bias, k, renorm):
    T, H = x_bits.shape
    E = Wr.shape[0]
    x = torch.from_numpy(x_bits.view(np.int16)).to(dev)
    w = torch.from_numpy(Wr).to(dev)
    b = torch.from_numpy(bias).to(dev)
    logits = torch.empty((T, E), dtype=torch.float32, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    gate = torch.empty((T, k), dtype=torch.float32, device=dev)
    cfg = B.pw_route_cfg(k=k, renorm=int(renorm), policy=0, threshold=0.15, critical_n=32)
    B.check(B.pw_route_topk(x.data_ptr(), w.data_ptr(), b.data_ptr(), T, H, E, cfg,
                            logits.data_ptr(), idx.data_ptr(), gate.data_ptr(), _stream(torch)))
    return logits.cpu().numpy(), idx.cpu().numpy(), gate.cpu().numpy()


def _check_route(lg, ig, gg, x_bits, Wr, bias, k, renorm):
    lo = orouter.router_logits(x_bits, Wr, bias)
    ulps = np.abs(lg.view(np.int32).astype(np.int64) - lo.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1
    assert (ulps == 0).mean() > 0.999          # float64 accumulation: virtually all identical
    io, go, _ = orouter.softmax_topk(lo, k, renorm)
    if not np.array_equal(lg, lo):             # only a 1-ulp logit could move a near tie
        io2, _, _ = orouter.softmax_topk(lg, k, renorm)
        assert np.array_equal(ig, io2)
    assert np.array_equal(ig, io)
    assert np.max(np.abs(gg - go)) <= GATE_ATOL


@pytest.mark.parametrize("name", list(CONFIGS))
def test_route_topk_full_size(torch_dev, name):
    torch, dev = torch_dev
    cfg = CONFIGS[name]
    for T in cfg.T_sweep:
        L = make_layer(cfg, T, with_weights=False)
        lg, ig, gg = _route_gpu(torch, dev, L.x_bf16, L.Wr, L.bias, cfg.k, cfg.renorm)
        _check_route(lg, ig, gg, L.x_bf16, L.Wr, L.bias, cfg.k, cfg.renorm)


@pytest.mark.parametrize("T,E,H,k,renorm", [(1, 8, 4096, 2, True), (5, 60, 200, 4, True),
                                            (33, 512, 64, 10, False), (3, 7, 33, 7, False),
                                            (2, 1024, 128, 16, True), (300, 64, 96, 8, False)])
def test_route_topk_shapes(torch_dev, T, E, H, k, renorm):
    torch, dev = torch_dev
    x_bits, Wr, bias = random_router_inputs(T, E, H, seed=T * E, zipf_s=1.2)
    lg, ig, gg = _route_gpu(torch, dev, x_bits, Wr, bias, k, renorm)
    _check_route(lg, ig, gg, x_bits, Wr, bias, k, renorm)


def test_route_all_equal_logits(torch_dev):
    torch, dev = torch_dev
    T, E, H, k = 4, 40, 64, 6
    x_bits = np.zeros((T, H), np.uint16)
    Wr = np.ones((E, H), np.float32)
    lg, ig, gg = _route_gpu(torch, dev, x_bits, Wr, np.zeros(E, np.float32), k, False)
    assert (lg == 0).all() and (ig == np.arange(k)).all()
    assert np.allclose(gg, 1.0 / E, rtol=0, atol=1e-9)


# ------------------------------------------------------------------ K3a / K3b
def _oracle_routed(cfg, T):
    L = make_layer(cfg, T, with_weights=False)
    lo = orouter.router_logits(L.x_bf16, L.Wr, L.bias)
    io, go, _ = orouter.softmax_topk(lo, cfg.k, cfg.renorm)
    return L, lo, io, go


def _substitute_gpu(torch, dev, lo, io, go, resident, k, policy, thr):
    T, E = lo.shape
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    l_d, i_d, g_d, r_d = t(lo), t(io), t(go), t(resident)
    act = torch.empty((T, k), dtype=torch.uint8, device=dev)
    mass = torch.empty((T,), dtype=torch.float32, device=dev)
    cfg = B.pw_route_cfg(k=k, renorm=1, policy=policy, threshold=thr, critical_n=0)
    B.check(B.pw_substitute(l_d.data_ptr(), i_d.data_ptr(), g_d.data_ptr(), r_d.data_ptr(), T, E,
                            cfg, act.data_ptr(), mass.data_ptr(), _stream(torch)))
    return i_d.cpu().numpy(), act.cpu().numpy(), mass.cpu().numpy()


@pytest.mark.parametrize("T", [1, 16, 64])
@pytest.mark.parametrize("policy,thr", [(1, 0.15), (2, 0.15), (0, 0.15), (1, float("inf"))])
def test_substitute_bit_exact(torch_dev, T, policy, thr):
    torch, dev = torch_dev
    cfg = CONFIGS["qwen3_next_80b_a3b"]
    L, lo, io, go = _oracle_routed(cfg, T)
    i2, act, m = _substitute_gpu(torch, dev, lo, io, go, L.resident, cfg.k, policy, thr)
    ie, ae, me, _ = opol.substitute(lo, io, go, L.resident, policy, thr)
    assert np.array_equal(i2, ie) and np.array_equal(act, ae)
    assert np.max(np.abs(m - me)) <= GATE_ATOL


def test_substitute_golden(torch_dev, golden):
    torch, dev = torch_dev
    g = golden("substitute_e6k3.json")
    lo = np.array(g["logits"], np.float32)
    io = np.array(g["idx"], np.int32)
    go = np.array(g["gate"], np.float32)
    res = np.array(g["resident"], np.uint8)
    for key, pol in (("threshold_rule", 1), ("first_choice", 2), ("fetch_all", 0)):
        i2, act, m = _substitute_gpu(torch, dev, lo, io, go, res, 3, pol, g["threshold"])
        assert i2.tolist() == g[key]["idx"] and act.tolist() == g[key]["action"], key
        assert np.allclose(m, g[key]["mass"], atol=1e-6), key


def _remap_gpu(torch, dev, lo, io, go, k, critical_n):
    T, E = lo.shape
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    l_d, i_d, g_d = t(lo), t(io), t(go)
    crit = torch.empty((E,), dtype=torch.uint8, device=dev)
    uniq = torch.full((2,), -1, dtype=torch.int32, device=dev)
    cfg = B.pw_route_cfg(k=k, renorm=0, policy=0, threshold=0.15, critical_n=critical_n)
    B.check(B.pw_remap(l_d.data_ptr(), i_d.data_ptr(), g_d.data_ptr(), T, E, cfg,
                       crit.data_ptr(), uniq.data_ptr(), _stream(torch)))
    i2 = i_d.cpu().numpy()
    # the distinct experts before / after the rewrite (the experts the FFN reads)
    assert uniq.cpu().tolist() == [len(np.unique(io)), len(np.unique(i2))]
    return i2, crit.cpu().numpy()


@pytest.mark.parametrize("T", [8, 32, 64])
@pytest.mark.parametrize("critical_n", [32, 8, 64])
def test_remap_bit_exact(torch_dev, T, critical_n):
    torch, dev = torch_dev
    cfg = CONFIGS["qwen2_57b_a14b"]
    L, lo, io, go = _oracle_routed(cfg, T)
    i2, crit = _remap_gpu(torch, dev, lo, io, go, cfg.k, critical_n)
    ie, ce = opol.remap(lo, io, go, critical_n)
    assert np.array_equal(crit, ce) and np.array_equal(i2, ie)
    for t in range(T):
        assert len(set(i2[t].tolist())) == cfg.k


def test_remap_golden(torch_dev, golden):
    torch, dev = torch_dev
    g = golden("remap_2tok.json")
    i2, crit = _remap_gpu(torch, dev, np.array(g["logits"], np.float32),
                          np.array(g["idx"], np.int32), np.array(g["gate"], np.float32), 3, 3)
    assert crit.tolist() == g["critical"] and i2.tolist() == g["idx_remapped"]


# ------------------------------------------------------------------ FFN (K2 + K4 + combine)
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


@pytest.mark.parametrize("name", list(SCALED))
def test_ffn_scaled_configs(torch_dev, name):
    torch, dev = torch_dev
    cfg = SCALED[name]
    T = max(cfg.T_sweep) if name != "mixtral" else 8
    L = make_layer(cfg, T)
    D = _device_layer(L)
    ref = olayer.route(L)
    y = _ffn_with(torch, D, ref["idx"], ref["gate"])
    yo, _ = offn.moe_ffn(L, ref["idx"], ref["gate"])
    assert_ffn_close(y, yo, name)


@pytest.mark.parametrize("q", [3, 4, 5, 6, 7, 8])
def test_ffn_every_bitwidth_via_commit(torch_dev, q):
    torch, dev = torch_dev
    cfg = SCALED["mixtral"]
    L = make_layer(cfg, 4)
    D = _device_layer(L)
    D.commit(list(range(2 * cfg.E)), [q] * (2 * cfg.E))
    qq = np.full((cfg.E, 2), q, np.uint8)
    assert (D.committed_bits() == q).all()
    ref = olayer.route(L)
    y = _ffn_with(torch, D, ref["idx"], ref["gate"])
    yo, _ = offn.moe_ffn(L, ref["idx"], ref["gate"], q=qq)
    assert_ffn_close(y, yo, f"q={q}")


def test_ffn_many_tokens_one_expert_and_empty_experts(torch_dev):
    torch, dev = torch_dev
    cfg = SCALED["qwen15"]
    T = 9
    L = make_layer(cfg, T)
    D = _device_layer(L)
    idx = np.array([[5, 7, 0, 59]] * T, np.int32)       # 9 tokens on 4 experts, 56 idle
    gate = np.tile(np.array([[0.4, 0.3, 0.2, 0.1]], np.float32), (T, 1))
    y = _ffn_with(torch, D, idx, gate)
    yo, _ = offn.moe_ffn(L, idx, gate)
    assert_ffn_close(y, yo, "9 tokens per expert")


def test_ffn_ragged_small_shapes(torch_dev):
    torch, dev = torch_dev
    cfg = CONFIGS["tiny"].scaled(H=128, I=128, E=3)
    L = make_layer(cfg, 1)
    D = _device_layer(L)
    idx = np.array([[2, 0]], np.int32)
    gate = np.array([[0.75, 0.25]], np.float32)
    y = _ffn_with(torch, D, idx, gate)
    yo, _ = offn.moe_ffn(L, idx, gate)
    assert_ffn_close(y, yo, "H=I=128")


# ------------------------------------------------------------------ whole layer
@pytest.mark.parametrize("name", list(SCALED))
def test_layer_end_to_end_scaled(torch_dev, name):
    torch, dev = torch_dev
    cfg = SCALED[name]
    T = min(cfg.T_sweep)
    L = make_layer(cfg, T)
    D = _device_layer(L)
    D.forward()
    ref = olayer.moe_layer(L)
    assert np.array_equal(D.idx.cpu().numpy(), ref["idx"])
    if "action" in ref:
        assert np.array_equal(D.action.cpu().numpy(), ref["action"])
    if "critical" in ref:
        assert np.array_equal(D.critical.cpu().numpy(), ref["critical"])
    assert_ffn_close(D.y.cpu().numpy(), ref["y"], name)
    assert D.status() == B.PW_OK


def test_layer_mixtral_full_size_batch1(torch_dev):
    torch, dev = torch_dev
    L = make_layer(CONFIGS["mixtral_8x7b"], 1)
    D = _device_layer(L)
    D.forward()
    ref = olayer.moe_layer(L)
    assert np.array_equal(D.idx.cpu().numpy(), ref["idx"])
    assert_ffn_close(D.y.cpu().numpy(), ref["y"], "mixtral T=1")
    assert D.status() == B.PW_OK


# ------------------------------------------------------------------ device-side errors
def test_non_resident_block_reports_and_zeroes(torch_dev):
    torch, dev = torch_dev
    cfg = CONFIGS["tiny"]
    L = make_layer(cfg, 4)
    D = _device_layer(L)
    idx = np.array([[1, 2]] * 4, np.int32)
    gate = np.array([[0.5, 0.5]] * 4, np.float32)
    D.set_state(2, MOD_DOWN, B.PW_PAGE_CPU)
    i_d = torch.from_numpy(idx).to(dev)
    g_d = torch.from_numpy(gate).to(dev)
    D.ffn(idx_ptr=i_d.data_ptr(), gate_ptr=g_d.data_ptr())
    assert D.status() == B.PW_ERR_NOT_RESIDENT
    y = D.y.cpu().numpy()
    _, out = offn.moe_ffn(L, idx, gate)
    y1 = 0.5 * out[np.arange(4) * 2]                     # expert 2's contribution is zero
    assert_ffn_close(y, y1, "expert 2 skipped")
    assert D.status() == B.PW_OK                          # status was cleared


def test_commit_out_of_range_is_refused(torch_dev):
    torch, dev = torch_dev
    L = make_layer(CONFIGS["tiny"], 4)
    D = _device_layer(L)
    before = D.committed_bits().copy()
    D.commit([0, 1], [2, 5])          # 2 < min_bits, 5 > parent bits (4)
    assert D.status() == B.PW_ERR_BAD_BITS
    assert np.array_equal(D.committed_bits(), before)
    D.commit([3], [3])
    assert D.status() == B.PW_OK and D.committed_bits()[1, 1] == 3


def test_bad_expert_id_reports(torch_dev):
    torch, dev = torch_dev
    L = make_layer(CONFIGS["tiny"], 4)
    D = _device_layer(L)
    idx = np.array([[1, 9]] * 4, np.int32)     # 9 >= E
    gate = np.array([[0.5, 0.5]] * 4, np.float32)
    i_d = torch.from_numpy(idx).to(dev)
    g_d = torch.from_numpy(gate).to(dev)
    D.ffn(idx_ptr=i_d.data_ptr(), gate_ptr=g_d.data_ptr())
    assert D.status() == B.PW_ERR_BAD_EXPERT
    _, out = offn.moe_ffn(L, np.array([[1, 1]] * 4, np.int32), gate)
    assert_ffn_close(D.y.cpu().numpy(), 0.5 * out[np.arange(4) * 2], "bad id contributes 0")
