"""ctypes binding of libpw (include/pw.h): the same entry points, same names, same arguments.

Pointers are passed as Python ints (device addresses, e.g. ``tensor.data_ptr()``) and streams as
raw ``cudaStream_t`` values (``torch.cuda.current_stream().cuda_stream``).  Every function
returns the ``pw_status`` code as an int; ``check()`` turns a non-zero code into ``PwError``.
There is no fallback: if ``libpw.so`` is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# PW_LIB_VARIANT=debug loads the debug build (device bounds checks, PW_ERR_BOUNDS)
LIB_PATH = os.path.join(HERE, "libpw_debug.so" if os.environ.get("PW_LIB_VARIANT") == "debug"
                        else "libpw.so")

PW_OK = 0
PW_ERR_INVALID_ARG = 1
PW_ERR_UNSUPPORTED = 2
PW_ERR_CUDA = 3
PW_ERR_NOT_RESIDENT = 4
PW_ERR_TIMEOUT = 5
PW_ERR_BAD_EXPERT = 6
PW_ERR_BAD_BITS = 7
PW_ERR_BOUNDS = 8

PW_MOD_GATE_UP = 0
PW_MOD_DOWN = 1
PW_LAYOUT_ROWS, PW_LAYOUT_TILED_GATE_UP, PW_LAYOUT_TILED_DOWN = 0, 1, 2
PW_PAGE_GPU, PW_PAGE_CPU, PW_PAGE_XFER = 0, 1, 2
PW_POLICY_FETCH_ALL, PW_POLICY_THRESHOLD, PW_POLICY_FIRST_CHOICE = 0, 1, 2
PW_ACT_HIT, PW_ACT_FETCH, PW_ACT_SUBST = 0, 1, 2
PW_MIN_BITS = 3
PW_MAX_BITS = 8
PW_MAX_EXPERTS = 1024
PW_MAX_TOPK = 16
PW_MAX_TOKENS = 4096

# every symbol include/pw.h declares
EXPORTS = ("pw_block_prepare", "pw_pack_bitplanes", "pw_route_topk", "pw_topk", "pw_substitute",
           "pw_remap", "pw_affinity_default", "pw_affinity_remap", "pw_cache_step", "pw_page_copy", "pw_page_update",
           "pw_plan_bitwidths",
           "pw_moe_workspace_bytes",
           "pw_moe_anyprec_forward",
           "pw_moe_anyprec_forward_static", "pw_set_tc_min_tokens", "pw_set_ffn_grid",
           "pw_set_wait_limit_ns", "pw_test_hold_down_items", "pw_commit_bits",
           "pw_get_status",
           "pw_status_string", "pw_version")
PW_STATIC_WORKSPACE_BYTES = 16 << 20


class PwError(RuntimeError):
    def __init__(self, code: int, where: str = ""):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({code})")


class pw_block(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_uint32), ("cols", ctypes.c_uint32),
                ("parent_bits", ctypes.c_uint8), ("min_bits", ctypes.c_uint8),
                ("desired_bits", ctypes.c_uint8), ("committed_bits", ctypes.c_uint8),
                ("state", ctypes.c_uint8), ("layout", ctypes.c_uint8),
                ("stored_bits", ctypes.c_uint8), ("reserved0", ctypes.c_uint8 * 1),
                ("planes", ctypes.c_void_p), ("lut", ctypes.c_void_p * 9),
                ("reserved1", ctypes.c_uint8 * 160)]


class pw_page_table(ctypes.Structure):
    _fields_ = [("num_layers", ctypes.c_uint32), ("num_experts", ctypes.c_uint32),
                ("blocks", ctypes.c_void_p)]


class pw_route_cfg(ctypes.Structure):
    _fields_ = [("k", ctypes.c_int32), ("renorm", ctypes.c_int32), ("policy", ctypes.c_int32),
                ("threshold", ctypes.c_float), ("critical_n", ctypes.c_int32)]


class pw_affinity_cfg(ctypes.Structure):
    _fields_ = [("num_bins", ctypes.c_int32), ("low_bins", ctypes.c_int32),
                ("bin_width", ctypes.c_double)]


assert ctypes.sizeof(pw_affinity_cfg) == 16
assert ctypes.sizeof(pw_block) == 256 and pw_block.layout.offset == 13
assert ctypes.sizeof(pw_page_table) == 16 and ctypes.sizeof(pw_route_cfg) == 20

_lib = None


def lib() -> ctypes.CDLL:
    """Load libpw.so (built in-tree); raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libpw.so not found at {LIB_PATH}; build it first "
                               "(python -c 'import __graft_entry__ as g; g.build()')")
        L = ctypes.CDLL(LIB_PATH)
        P, I, Z, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
        L.pw_block_prepare.argtypes = [ctypes.POINTER(pw_block)]
        L.pw_pack_bitplanes.argtypes = [P, I, I, I, I, P, S]
        L.pw_route_topk.argtypes = [P, P, P, I, I, I, ctypes.POINTER(pw_route_cfg), P, P, P, S]
        L.pw_topk.argtypes = [P, I, I, ctypes.POINTER(pw_route_cfg), P, P, S]
        L.pw_substitute.argtypes = [P, P, P, P, I, I, ctypes.POINTER(pw_route_cfg), P, P, S]
        L.pw_remap.argtypes = [P, P, P, I, I, ctypes.POINTER(pw_route_cfg), P, P, S]
        L.pw_affinity_default.argtypes = [I, I, ctypes.POINTER(pw_affinity_cfg)]
        L.pw_cache_step.argtypes = [P, P, P, I, I, ctypes.POINTER(pw_route_cfg), ctypes.c_double,
                                    P, P, P, I, P, P, P, S]
        L.pw_affinity_remap.argtypes = [P, P, P, I, I, ctypes.POINTER(pw_route_cfg),
                                        ctypes.POINTER(pw_affinity_cfg), P, P, P, S]
        L.pw_moe_workspace_bytes.argtypes = [I, I, I, I, I]
        L.pw_moe_workspace_bytes.restype = Z
        L.pw_moe_anyprec_forward.argtypes = [P, I, I, P, I, I, I, I, P, P, P, P, Z, S]
        L.pw_moe_anyprec_forward_static.argtypes = [P, I, I, P, I, I, I, I, P, P, P, S]
        L.pw_set_tc_min_tokens.argtypes = [I]
        L.pw_set_ffn_grid.argtypes = [I]
        L.pw_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
        L.pw_test_hold_down_items.argtypes = [I]
        L.pw_commit_bits.argtypes = [P, I, P, P, I, S]
        L.pw_page_copy.argtypes = [P, I, P, I, I, I, I, S]
        L.pw_page_update.argtypes = [P, I, P, I, S]
        L.pw_plan_bitwidths.argtypes = [I, P, P, P, P, ctypes.c_uint64, P]
        L.pw_get_status.argtypes = [S]
        L.pw_status_string.argtypes = [I]
        L.pw_status_string.restype = ctypes.c_char_p
        L.pw_version.restype = ctypes.c_char_p
        for name in EXPORTS:
            fn = getattr(L, name)
            if name not in ("pw_moe_workspace_bytes", "pw_status_string", "pw_version"):
                fn.restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(code: int) -> str:
    try:
        return lib().pw_status_string(int(code)).decode()
    except Exception:  # library missing: still give a readable error
        return f"status {code}"


def check(code: int, where: str = "libpw") -> None:
    if code != PW_OK:
        raise PwError(code, where)


def _cfg(cfg):
    return ctypes.byref(cfg) if cfg is not None else None


def pw_version() -> str:
    return lib().pw_version().decode()


def pw_status_string(code: int) -> str:
    return lib().pw_status_string(int(code)).decode()


def pw_block_prepare(blk: pw_block) -> int:
    return lib().pw_block_prepare(ctypes.byref(blk))


def pw_pack_bitplanes(idx, rows, cols, n, layout, planes, stream=0) -> int:
    return lib().pw_pack_bitplanes(idx, rows, cols, n, layout, planes, stream)


def pw_route_topk(x_bf16, Wr, bias, T, H, E, cfg, logits, idx, gate, stream=0) -> int:
    return lib().pw_route_topk(x_bf16, Wr, bias, T, H, E, _cfg(cfg), logits, idx, gate, stream)


def pw_topk(logits, T, E, cfg, idx, gate, stream=0) -> int:
    return lib().pw_topk(logits, T, E, _cfg(cfg), idx, gate, stream)


def pw_substitute(logits, idx, gate, resident, T, E, cfg, action, mass, stream=0) -> int:
    return lib().pw_substitute(logits, idx, gate, resident, T, E, _cfg(cfg), action, mass, stream)


def pw_remap(logits, idx, gate, T, E, cfg, critical, unique=0, stream=0) -> int:
    """unique: device int32[2] receiving the distinct experts before / after (0 = none)."""
    return lib().pw_remap(logits, idx, gate, T, E, _cfg(cfg), critical, unique, stream)


def pw_affinity_default(E, k, out) -> int:
    return lib().pw_affinity_default(E, k, _cfg(out))


def pw_affinity_remap(logits, idx, gate, T, E, cfg, acfg, critical, bins, unique=0,
                      stream=0) -> int:
    return lib().pw_affinity_remap(logits, idx, gate, T, E, _cfg(cfg), _cfg(acfg), critical,
                                   bins, unique, stream)


def pw_cache_step(logits, idx, gate, T, E, cfg, beta, resident, mass, freq, capacity, action,
                  mass_t, stats, stream=0) -> int:
    return lib().pw_cache_step(logits, idx, gate, T, E, _cfg(cfg), float(beta), resident, mass,
                               freq, capacity, action, mass_t, stats, stream)


def pw_moe_workspace_bytes(T, k, E, H, I) -> int:
    return int(lib().pw_moe_workspace_bytes(T, k, E, H, I))


def pw_moe_anyprec_forward(pt_dev, layer, E, x_bf16, T, H, I, k, idx, gate, y, workspace,
                           ws_bytes, stream=0) -> int:
    return lib().pw_moe_anyprec_forward(pt_dev, layer, E, x_bf16, T, H, I, k, idx, gate, y,
                                        workspace, ws_bytes, stream)


def pw_moe_anyprec_forward_static(pt_dev, layer, E, x_bf16, T, H, I, k, idx, gate, y,
                                  stream=0) -> int:
    """pw_moe_anyprec_forward with libpw's own fixed scratch array instead of a caller
    workspace, for callers that cannot allocate device memory (see include/pw.h)."""
    return lib().pw_moe_anyprec_forward_static(pt_dev, layer, E, x_bf16, T, H, I, k, idx, gate,
                                               y, stream)


def pw_set_tc_min_tokens(tokens_per_expert) -> int:
    return lib().pw_set_tc_min_tokens(tokens_per_expert)


def pw_set_ffn_grid(ctas) -> int:
    """Test hook: CTAs of the FFN launch (0 = one per SM)."""
    return lib().pw_set_ffn_grid(ctas)


def pw_set_wait_limit_ns(ns) -> int:
    """Test hook: bound of the kernels' spin waits on the current device (0 = default 2 s)."""
    return lib().pw_set_wait_limit_ns(int(ns))


def pw_test_hold_down_items(extra) -> int:
    """Test hook: down items wait for `extra` gate_up completions that never come (0 = off)."""
    return lib().pw_test_hold_down_items(extra)


def pw_commit_bits(pt_dev, num_blocks, block_ids, q, count, stream=0) -> int:
    return lib().pw_commit_bits(pt_dev, num_blocks, block_ids, q, count, stream)


def pw_page_copy(src, src_bits, dst, dst_bits, rows, cols, q, stream=0) -> int:
    return lib().pw_page_copy(src, src_bits, dst, dst_bits, rows, cols, q, stream)


def pw_page_update(pt_dev, num_blocks, updates, count, stream=0) -> int:
    return lib().pw_page_update(pt_dev, num_blocks, updates, count, stream)


def pw_plan_bitwidths(nblocks, damage, bytes_, qmin, qmax, budget, q_out) -> int:
    """Host arrays as integer addresses (e.g. numpy arr.ctypes.data)."""
    return lib().pw_plan_bitwidths(nblocks, damage, bytes_, qmin, qmax, int(budget), q_out)


class pw_page_update_t(ctypes.Structure):
    _fields_ = [("block", ctypes.c_int32), ("state", ctypes.c_uint8),
                ("stored_bits", ctypes.c_uint8), ("committed_bits", ctypes.c_uint8),
                ("reserved", ctypes.c_uint8), ("planes", ctypes.c_void_p)]


assert ctypes.sizeof(pw_page_update_t) == 16


def pw_get_status(stream=0) -> int:
    return lib().pw_get_status(stream)
