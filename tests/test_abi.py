"""The C ABI on the host: the library loads, exports every function include/pw.h declares, and
rejects bad arguments before launching anything (no GPU needed for these calls)."""
import ctypes
import os
import re

from any_precision_expert_pw_b200 import binding as B
from conftest import ROOT


def _declared():
    src = open(os.path.join(ROOT, "include", "pw.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pw_[a-z_]+)\s*\(", src)))


def test_header_and_binding_agree(libpw):
    declared = _declared()
    assert declared == sorted(B.EXPORTS)
    for name in declared:
        assert hasattr(libpw, name), name


def test_debug_build_exports_the_same_functions(libpw):
    # libpw_debug.so: the same C ABI with device bounds checks (PW_ERR_BOUNDS)
    path = os.path.join(os.path.dirname(B.LIB_PATH), "libpw_debug.so")
    dbg = ctypes.CDLL(path)
    for name in _declared():
        assert hasattr(dbg, name), name
    dbg.pw_version.restype = ctypes.c_char_p
    assert b"debug" in dbg.pw_version() and b"sm_100a" in dbg.pw_version()
    dbg.pw_status_string.restype = ctypes.c_char_p
    assert dbg.pw_status_string(B.PW_ERR_BOUNDS) == b"PW_ERR_BOUNDS"
    assert B.pw_status_string(B.PW_ERR_BOUNDS) == "PW_ERR_BOUNDS"


def test_status_strings_and_version(libpw):
    assert B.pw_status_string(B.PW_OK) == "PW_OK"
    assert B.pw_status_string(B.PW_ERR_BAD_BITS) == "PW_ERR_BAD_BITS"
    assert "sm_100a" in B.pw_version()


def test_struct_layouts():
    assert ctypes.sizeof(B.pw_block) == 256
    assert B.pw_block.planes.offset == 16 and B.pw_block.lut.offset == 24
    assert B.pw_block.layout.offset == 13 and B.pw_block.reserved1.offset == 96


def test_host_argument_checks(libpw):
    cfg = B.pw_route_cfg(k=2, renorm=1, policy=1, threshold=0.15, critical_n=32)
    bad = B.PW_ERR_INVALID_ARG
    rows_l, tiled = B.PW_LAYOUT_ROWS, B.PW_LAYOUT_TILED_DOWN
    assert B.pw_pack_bitplanes(0, 4, 64, 4, rows_l, 0) == bad
    assert B.pw_pack_bitplanes(16, 4, 33, 4, rows_l, 16) == bad           # ragged columns
    assert B.pw_pack_bitplanes(16, 4, 64, 9, rows_l, 16) == bad           # n > 8
    assert B.pw_pack_bitplanes(16, 32, 128, 4, 3, 16) == bad              # unknown layout
    assert B.pw_pack_bitplanes(16, 48, 128, 4, tiled, 16) == bad          # rows % 32
    assert B.pw_pack_bitplanes(16, 32, 96, 4, tiled, 16) == bad           # cols % 128
    assert B.pw_route_topk(16, 16, 0, 0, 64, 8, cfg, 16, 16, 16) == bad      # T = 0
    assert B.pw_route_topk(16, 16, 0, 4, 64, 2000, cfg, 16, 16, 16) == bad   # E too large
    cfg.k = 9
    assert B.pw_route_topk(16, 16, 0, 4, 64, 8, cfg, 16, 16, 16) == bad      # k > E
    cfg.k = 2
    cfg.policy = 7
    assert B.pw_substitute(16, 16, 16, 16, 4, 8, cfg, 0, 0) == bad           # unknown policy
    cfg.policy = 1
    cfg.critical_n = -1
    assert B.pw_remap(16, 16, 16, 4, 8, cfg, 0) == bad
    ws = B.pw_moe_workspace_bytes(4, 2, 8, 256, 512)
    assert ws > 0 and B.pw_moe_workspace_bytes(0, 2, 8, 256, 512) == 0
    fwd = B.pw_moe_anyprec_forward
    assert fwd(256, 0, 8, 256, 4, 256, 512, 2, 256, 256, 256, 256, ws - 1) == bad  # small ws
    assert fwd(256, 0, 8, 256, 4, 200, 512, 2, 256, 256, 256, 256, ws) == bad      # H % 128
    assert fwd(256, 0, 8, 256, 4, 256, 512, 2, 256, 256, 256, 258, ws) == bad      # ws align
    assert B.pw_commit_bits(0, 16, 16, 16, 1) == bad


def test_affinity_defaults_and_argument_checks(libpw):
    import math
    from oracle.affinity import default_bins
    for E, k in ((64, 8), (8, 2), (512, 10), (60, 4), (4, 4), (1, 1)):
        a = B.pw_affinity_cfg()
        assert B.pw_affinity_default(E, k, a) == B.PW_OK
        nb, w, low = default_bins(E, k)
        assert (a.num_bins, a.low_bins) == (nb, low)
        assert (math.isinf(a.bin_width) and math.isinf(w)) or a.bin_width == w
    bad = B.PW_ERR_INVALID_ARG
    assert B.pw_affinity_default(8, 9, B.pw_affinity_cfg()) == bad
    cfg = B.pw_route_cfg(k=2, renorm=1, policy=1, threshold=0.15, critical_n=4)
    for a in (B.pw_affinity_cfg(0, 1, 0.5), B.pw_affinity_cfg(4, 2, 0.0),
              B.pw_affinity_cfg(4, 2, float("nan")), B.pw_affinity_cfg(4, -1, 0.5)):
        assert B.pw_affinity_remap(16, 16, 16, 4, 8, cfg, a, 0, 0, 0) == bad
    assert B.pw_affinity_remap(16, 16, 16, 4, 8, cfg, None, 0, 0, 0) == bad


def test_block_prepare_rejects_bad_blocks(libpw):
    blk = B.pw_block()
    assert B.pw_block_prepare(blk) == B.PW_ERR_INVALID_ARG                 # no planes
    blk.planes, blk.rows, blk.cols, blk.parent_bits, blk.min_bits = 4096, 64, 100, 8, 3
    assert B.pw_block_prepare(blk) == B.PW_ERR_INVALID_ARG                 # cols % 128
    blk.cols = 128
    assert B.pw_block_prepare(blk) == B.PW_ERR_INVALID_ARG                 # LUTs missing
    for b in range(3, 9):
        blk.lut[b] = 4096 * (b + 1)
    blk.committed_bits = 2
    assert B.pw_block_prepare(blk) == B.PW_ERR_INVALID_ARG                 # q below min_bits
    blk.committed_bits = 5
    assert B.pw_block_prepare(blk) == B.PW_ERR_INVALID_ARG                 # rows layout
    blk.layout = B.PW_LAYOUT_TILED_GATE_UP
    assert B.pw_block_prepare(blk) == B.PW_OK                              # host-only check
    blk.planes = 4096 + 8
    assert B.pw_block_prepare(blk) == B.PW_ERR_INVALID_ARG                 # planes alignment


def test_tc_switch_is_host_only(libpw):
    # the FFN path switch is plain host state: no device call, negative values refused
    assert B.pw_set_tc_min_tokens(0) == B.PW_OK
    assert B.pw_set_tc_min_tokens(1 << 20) == B.PW_OK
    assert B.pw_set_tc_min_tokens(-1) == B.PW_ERR_INVALID_ARG
    assert B.pw_set_tc_min_tokens(4) == B.PW_OK          # the library default


def test_workspace_holds_tensor_core_operands(libpw):
    # the workspace has room for both FFN paths: among the rest, the fp16 operands of the
    # tensor-core path, one row per padded position (each active expert's rows rounded up to 16):
    # x (H columns) and h as hi and lo parts (2 I columns)
    for T, k, E, H, I in [(1, 2, 8, 4096, 14336), (64, 8, 64, 3584, 2560), (4, 2, 8, 256, 512),
                          (512, 10, 512, 2048, 512)]:
        ws = B.pw_moe_workspace_bytes(T, k, E, H, I)
        tk = T * k
        rows_pad = tk + 15 * min(E, tk)
        kslices = min(8, max(1, -(-I // 512) // 2))  # the most k-slices of the down partials
        assert ws >= 2 * rows_pad * (H + 2 * I) + 4 * tk * H * kslices
        assert ws % 256 == 0
