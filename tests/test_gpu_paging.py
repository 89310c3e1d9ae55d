"""Page movement on the GPU: pw_page_copy (top-q planes between tiled buffers with different
planes per run, host <-> device and device <-> device), pw_page_update (stream-ordered page
table edits: XFER while moving, compact paged-in blocks), and a forward over blocks that keep
only their top q planes on the device, each against the oracle."""
import numpy as np
import pytest

from any_precision_expert_pw_b200 import binding as B
from any_precision_expert_pw_b200.inputs import MOD_DOWN, MOD_GATE_UP, make_layer, random_indices
from gpu_helpers import SCALED, assert_ffn_close, tiled_reference
from oracle import bitplanes as obp
from oracle import ffn as offn
from oracle import layer as olayer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_dev(libpw):
    import torch
    return torch, torch.device("cuda:0")


def _st(torch):
    return torch.cuda.current_stream().cuda_stream


@pytest.mark.parametrize("rows,cols,layout", [(96, 4096, B.PW_LAYOUT_TILED_DOWN),
                                              (64, 1408, B.PW_LAYOUT_TILED_GATE_UP),
                                              (32, 512, B.PW_LAYOUT_TILED_DOWN)])
@pytest.mark.parametrize("q", [3, 5, 8])
def test_page_copy_round_trip(torch_dev, rows, cols, layout, q):
    torch, dev = torch_dev
    n = 8
    idx = random_indices(rows, cols, n, seed=rows * 7 + cols + q)
    words = rows * cols // 32
    full = torch.empty((n * words,), dtype=torch.int32, device=dev)
    B.check(B.pw_pack_bitplanes(torch.from_numpy(idx).to(dev).data_ptr(), rows, cols, n, layout,
                                full.data_ptr(), _st(torch)))
    ref = obp.pack_bitplanes(idx, n)
    # device (8 per run) -> pinned host (8 per run) -> device (q per run)
    host = torch.empty((n * words,), dtype=torch.int32).pin_memory()
    B.check(B.pw_page_copy(full.data_ptr(), n, host.data_ptr(), n, rows, cols, n, _st(torch)))
    comp = torch.full((q * words,), -1, dtype=torch.int32, device=dev)
    B.check(B.pw_page_copy(host.data_ptr(), n, comp.data_ptr(), q, rows, cols, q, _st(torch)))
    torch.cuda.synchronize()
    assert np.array_equal(host.numpy().view(np.uint32), tiled_reference(ref, layout))
    assert np.array_equal(comp.cpu().numpy().view(np.uint32), tiled_reference(ref[:q], layout))
    # device (q per run) -> device (8 per run), top q planes only: the rest stays as it was
    back = torch.zeros((n * words,), dtype=torch.int32, device=dev)
    B.check(B.pw_page_copy(comp.data_ptr(), q, back.data_ptr(), n, rows, cols, q, _st(torch)))
    want = tiled_reference(np.concatenate([ref[:q], np.zeros_like(ref[q:])]), layout)
    assert np.array_equal(back.cpu().numpy().view(np.uint32), want)


def _paged_layer(torch):
    L = make_layer(SCALED["mixtral"], 2)
    from any_precision_expert_pw_b200.device_layer import DeviceLayer
    D = DeviceLayer(L)
    return L, D


def test_forward_over_compact_paged_blocks(torch_dev):
    torch, dev = torch_dev
    L, D = _paged_layer(torch)
    n = L.cfg.n
    ref = olayer.route(L)
    used = sorted(set(ref["idx"].reshape(-1).tolist()))
    keep, ups = [], []
    q_new = np.array(L.q, copy=True)
    for e in used:
        for m in (MOD_GATE_UP, MOD_DOWN):
            R, C = L.block_shape(m)
            q = 3 + (e + m) % 3                              # page in at 3, 4 or 5 bits
            q_new[e, m] = q
            comp = torch.empty((q * R * C // 32,), dtype=torch.int32, device=dev)
            B.check(B.pw_page_copy(D.planes[(e, m)].data_ptr(), n, comp.data_ptr(), q, R, C, q,
                                   D.stream))
            keep.append(comp)
            ups.append({"block": e * 2 + m, "state": B.PW_PAGE_GPU, "stored_bits": q,
                        "committed_bits": q, "planes": comp.data_ptr()})
    D.page_update(ups)
    D.forward()
    assert D.status() == B.PW_OK
    blocks = D.blocks_dev.view(-1, 256).cpu().numpy()
    for e in used:
        for m in (MOD_GATE_UP, MOD_DOWN):
            assert blocks[e * 2 + m, 14] == q_new[e, m] == blocks[e * 2 + m, 11]
    yo, _ = offn.moe_ffn(L, ref["idx"], ref["gate"], q=q_new)
    assert_ffn_close(D.y.cpu().numpy(), yo, "compact paged blocks")
    # a commit above the stored planes is refused; one within them is taken
    D.commit([used[0] * 2], [q_new[used[0], 0] + 1])
    assert D.status() == B.PW_ERR_BAD_BITS
    D.commit([used[0] * 2], [3])
    assert D.status() == B.PW_OK


def test_xfer_state_reads_as_not_resident(torch_dev):
    torch, dev = torch_dev
    L, D = _paged_layer(torch)
    ref = olayer.route(L)
    e = int(ref["idx"][0, 0])
    D.page_update([{"block": e * 2 + MOD_GATE_UP, "state": B.PW_PAGE_XFER}])
    D.forward()
    assert D.status() == B.PW_ERR_NOT_RESIDENT
    D.page_update([{"block": e * 2 + MOD_GATE_UP, "state": B.PW_PAGE_GPU}])
    D.forward()
    assert D.status() == B.PW_OK
    yo, _ = offn.moe_ffn(L, ref["idx"], ref["gate"])
    assert_ffn_close(D.y.cpu().numpy(), yo, "back to GPU")


def test_inconsistent_page_updates_are_refused(torch_dev):
    torch, dev = torch_dev
    L, D = _paged_layer(torch)
    before = D.blocks_dev.clone()
    D.page_update([{"block": 0, "stored_bits": 9},                 # above parent bits
                   {"block": 1, "stored_bits": 4, "committed_bits": 5},  # q above stored
                   {"block": 2, "state": 7},                        # no such state
                   {"block": 10 ** 6, "state": B.PW_PAGE_CPU}])     # no such block
    assert D.status() == B.PW_ERR_BAD_BITS
    assert torch.equal(D.blocks_dev, before)
