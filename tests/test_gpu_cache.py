"""Parity of pw_cache_step (expert cache across decode steps: Quality-First and Speed-First)
against the oracle over multi-step routing streams: the rewritten assignments, actions, the
resident set, the accumulated substituted mass (float64), the selection counts and the
per-step counts of fetches, admissions and evictions, all bit-exact at every step."""
import numpy as np
import pytest

from any_precision_expert_pw_b200 import binding as B
from any_precision_expert_pw_b200.inputs import logit_stream
from oracle import policy as op
from oracle.cache import CacheState, cache_step
from oracle.router import softmax_topk

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_dev(libpw):
    import torch
    return torch, torch.device("cuda:0")


def _run(torch, E, k, T, steps, cap, policy, thr, beta, seed):
    dev = torch.device("cuda:0")
    stream = logit_stream(E, T, steps, seed=seed, topic_len=8)
    rng = np.random.default_rng(seed)
    res0 = np.zeros(E, np.uint8)
    res0[rng.choice(E, cap, replace=False)] = 1
    st = CacheState(res0)
    d_res = torch.from_numpy(res0.copy()).to(dev)
    d_mass = torch.zeros(E, dtype=torch.float64, device=dev)
    d_freq = torch.zeros(E, dtype=torch.int32, device=dev)
    d_act = torch.empty((T, k), dtype=torch.uint8, device=dev)
    d_m = torch.empty((T,), dtype=torch.float32, device=dev)
    d_stats = torch.zeros(3, dtype=torch.int32, device=dev)
    cfg = B.pw_route_cfg(k=k, renorm=1, policy=policy, threshold=thr, critical_n=0)
    cs = torch.cuda.current_stream().cuda_stream
    totals = np.zeros(3, np.int64)
    for s, lo in enumerate(stream):
        idx, g, _ = softmax_topk(lo, k, True)
        d_lo = torch.from_numpy(lo).to(dev)
        d_idx = torch.from_numpy(idx.copy()).to(dev)
        d_g = torch.from_numpy(g).to(dev)
        B.check(B.pw_cache_step(d_lo.data_ptr(), d_idx.data_ptr(), d_g.data_ptr(), T, E, cfg,
                                beta, d_res.data_ptr(), d_mass.data_ptr(), d_freq.data_ptr(), cap,
                                d_act.data_ptr(), d_m.data_ptr(), d_stats.data_ptr(), cs),
                "pw_cache_step")
        i2, act, m32, nf, na, nev = cache_step(st, lo, idx, g, policy, thr, beta)
        assert np.array_equal(d_idx.cpu().numpy(), i2), f"step {s}"
        assert np.array_equal(d_act.cpu().numpy(), act), f"step {s}"
        assert np.array_equal(d_m.cpu().numpy(), m32), f"step {s}"
        assert np.array_equal(d_res.cpu().numpy(), st.resident), f"step {s}"
        assert np.array_equal(d_mass.cpu().numpy(), st.mass), f"step {s}"
        assert np.array_equal(d_freq.cpu().numpy().astype(np.int64), st.freq), f"step {s}"
        assert d_stats.cpu().numpy().tolist() == [nf, na, nev], f"step {s}"
        totals += (nf, na, nev)
    assert B.pw_get_status(cs) == B.PW_OK
    return totals


@pytest.mark.parametrize("T", [1, 16])
@pytest.mark.parametrize("name,policy", [("quality-first", op.POLICY_THRESHOLD),
                                         ("speed-first", op.POLICY_FIRST_CHOICE)])
def test_cache_stream_qwen3_next_shaped(torch_dev, T, name, policy):
    torch, _ = torch_dev
    totals = _run(torch, 512, 10, T, 40, 128, policy, 0.15, 0.5, seed=T + policy)
    assert totals[0] > 0 and totals[2] > 0                      # the stream exercises both


def test_cache_insertions_beyond_capacity(torch_dev):
    torch, _ = torch_dev
    # capacity 4 with 16 tokens x top-4 of 32 experts: insertions exceed the capacity
    _run(torch, 32, 4, 16, 12, 4, op.POLICY_FETCH_ALL, 0.15, 0.5, seed=9)


def test_cache_all_resident_and_infinite_beta(torch_dev):
    torch, _ = torch_dev
    t = _run(torch, 64, 8, 4, 10, 64, op.POLICY_THRESHOLD, 0.15, 0.5, seed=3)
    assert t.tolist() == [0, 0, 0]
    t = _run(torch, 64, 8, 4, 10, 16, op.POLICY_FIRST_CHOICE, 0.15, float("inf"), seed=4)
    assert t[1] == 0


@pytest.mark.parametrize("E,k,T,renorm", [(512, 10, 16, True), (64, 8, 33, False), (8, 2, 5, True)])
def test_topk_from_logits(torch_dev, E, k, T, renorm):
    torch, dev = torch_dev
    lo = logit_stream(E, T, 1, seed=E + k, topic_len=1)[0]
    d_lo = torch.from_numpy(lo).to(dev)
    d_idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    d_g = torch.empty((T, k), dtype=torch.float32, device=dev)
    cfg = B.pw_route_cfg(k=k, renorm=int(renorm), policy=0, threshold=0.15, critical_n=0)
    cs = torch.cuda.current_stream().cuda_stream
    B.check(B.pw_topk(d_lo.data_ptr(), T, E, cfg, d_idx.data_ptr(), d_g.data_ptr(), cs))
    idx, g, _ = softmax_topk(lo, k, renorm)
    assert np.array_equal(d_idx.cpu().numpy(), idx)
    assert np.max(np.abs(d_g.cpu().numpy() - g)) <= 1e-6
