"""Parity of pw_affinity_remap (LYNX AffinityBinning, one reading of it) against the oracle:
bins, critical set and remapped indices bit-exact, on the Qwen2-57B-A14B-shaped and the
Qwen3-Next-80B-A3B-shaped routers, plus the reductions the reading implies (w = +inf gives
pw_remap, low_bins = 0 gives the identity)."""
import math

import numpy as np
import pytest

from any_precision_expert_pw_b200 import binding as B
from any_precision_expert_pw_b200.inputs import CONFIGS, make_layer
from oracle import affinity as oa
from oracle import policy as opol
from oracle import router as orouter

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_dev(libpw):
    import torch
    return torch, torch.device("cuda:0")


def _routed(name, T):
    cfg = CONFIGS[name]
    L = make_layer(cfg, T, with_weights=False)
    lo = orouter.router_logits(L.x_bf16, L.Wr, L.bias)
    io, go, _ = orouter.softmax_topk(lo, cfg.k, cfg.renorm)
    return cfg, lo, io, go


def _affinity_gpu(torch, lo, io, go, k, critical_n, nb, w, low):
    T, E = lo.shape
    dev = torch.device("cuda:0")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    l_d, i_d, g_d = t(lo), t(io), t(go)
    crit = torch.empty((E,), dtype=torch.uint8, device=dev)
    bins = torch.empty((T,), dtype=torch.int32, device=dev)
    uniq = torch.full((2,), -1, dtype=torch.int32, device=dev)
    cfg = B.pw_route_cfg(k=k, renorm=0, policy=0, threshold=0.15, critical_n=critical_n)
    acfg = B.pw_affinity_cfg(num_bins=nb, low_bins=low, bin_width=w)
    st = torch.cuda.current_stream().cuda_stream
    B.check(B.pw_affinity_remap(l_d.data_ptr(), i_d.data_ptr(), g_d.data_ptr(), T, E, cfg, acfg,
                                crit.data_ptr(), bins.data_ptr(), uniq.data_ptr(), st),
            "pw_affinity_remap")
    assert B.pw_get_status(st) == B.PW_OK
    i2 = i_d.cpu().numpy()
    assert uniq.cpu().tolist() == [len(np.unique(io)), len(np.unique(i2))]
    return i2, crit.cpu().numpy(), bins.cpu().numpy()


@pytest.mark.parametrize("name,T", [("qwen2_57b_a14b", 8), ("qwen2_57b_a14b", 32),
                                    ("qwen2_57b_a14b", 64), ("qwen3_next_80b_a3b", 16),
                                    ("mixtral_8x7b", 64)])
def test_affinity_remap_bit_exact(torch_dev, name, T):
    torch, _ = torch_dev
    cfg, lo, io, go = _routed(name, T)
    nb, w, low = oa.default_bins(cfg.E, cfg.k)
    acfg = B.pw_affinity_cfg()
    B.check(B.pw_affinity_default(cfg.E, cfg.k, acfg))
    assert (acfg.num_bins, acfg.low_bins, acfg.bin_width) == (nb, low, w)
    crit_n = min(cfg.critical_n, cfg.E)
    i2, crit, bins = _affinity_gpu(torch, lo, io, go, cfg.k, crit_n, nb, w, low)
    ie, ce, be, _ = oa.affinity_remap(lo, io, go, crit_n, nb, w, low)
    assert np.array_equal(bins, be)
    assert np.array_equal(crit, ce)
    assert np.array_equal(i2, ie)
    for t in range(T):
        assert len(set(i2[t].tolist())) == cfg.k


def test_infinite_width_is_pw_remap(torch_dev):
    torch, _ = torch_dev
    cfg, lo, io, go = _routed("qwen2_57b_a14b", 32)
    i2, crit, bins = _affinity_gpu(torch, lo, io, go, cfg.k, 32, 1, math.inf, 1)
    ie, ce = opol.remap(lo, io, go, 32)
    assert not bins.any()
    assert np.array_equal(crit, ce) and np.array_equal(i2, ie)


def test_no_low_bins_is_identity_and_sharp_tokens_kept(torch_dev):
    torch, _ = torch_dev
    cfg, lo, io, go = _routed("qwen2_57b_a14b", 64)
    nb, w, _ = oa.default_bins(cfg.E, cfg.k)
    i2, _, _ = _affinity_gpu(torch, lo, io, go, cfg.k, 32, nb, w, 0)
    assert np.array_equal(i2, io)
    # a batch where one token is sharply confident: its experts stay even if not critical
    lo2 = lo.copy()
    lo2[0, io[0, 0]] += 50.0
    io2, go2, _ = orouter.softmax_topk(lo2, cfg.k, cfg.renorm)
    nb, w, low = oa.default_bins(cfg.E, cfg.k)
    i3, _, b3 = _affinity_gpu(torch, lo2, io2, go2, cfg.k, 8, nb, w, low)
    assert b3[0] == nb - 1 and np.array_equal(i3[0], io2[0])


def test_hand_case(torch_dev):
    torch, _ = torch_dev
    logits = np.array([[3.0, 1.0, 0.5, 0.0, 0.0, 0.0],
                       [0.0, 1.2, 1.0, 0.0, 0.9, 0.0],
                       [0.0, 0.0, 2.0, 1.3, 0.0, 1.0]], dtype=np.float32)
    idx = np.array([[0, 1], [1, 2], [2, 3]], dtype=np.int32)
    gate = np.array([[0.6, 0.4], [0.5, 0.5], [0.7, 0.3]], dtype=np.float32)
    i2, crit, bins = _affinity_gpu(torch, logits, idx, gate, 2, 3, 4, 0.5, 2)
    assert bins.tolist() == [3, 0, 1]
    assert crit.tolist() == [1, 1, 1, 0, 0, 0]
    assert i2.tolist() == [[0, 1], [1, 2], [2, 0]]
