"""Runs the layer forward in a process of its own, with guard words around the output and
after the workspace, and checks that the kernels wrote inside their buffers only.

Called by test_gpu_debug_build.py once per library variant (PW_LIB_VARIANT=debug selects
libpw_debug.so, whose kernels check every index they derive from the grouping and record
PW_ERR_BOUNDS instead of reading or writing outside a buffer).  For each case: the output
y sits between two guard regions of NaN words with a fixed bit pattern, the workspace is
filled with 0xA5 bytes before the call (the forward must not rely on zeroed scratch) and
followed by a guard region of the same bytes; after the call the status must be PW_OK, both
guards intact, and y within the FFN tolerance of the oracle.  Prints one JSON line per case
and exits 1 on the first failure."""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

from any_precision_expert_pw_b200 import binding as B  # noqa: E402
from any_precision_expert_pw_b200.inputs import CONFIGS, make_layer  # noqa: E402
from gpu_helpers import FFN_RTOL_RMS, SCALED, ffn_err  # noqa: E402
from oracle import layer as olayer  # noqa: E402

GUARD_WORDS = 4096          # fp32 words before and after y
GUARD_BYTES = 1 << 16       # bytes after the workspace
Y_PATTERN = 0x7FC0DEAD      # a NaN with a payload no kernel writes
WS_PATTERN = 0xA5

# (shape, T, pw_set_tc_min_tokens value or None): both FFN paths on shapes with ragged column
# tails, a batch with several tensor-core passes per expert, and the Mixtral-shaped layer at
# full size at batch 1
CASES = [("tiny", 4, None), ("tiny", 4, 0), ("mixtral", 8, None), ("mixtral", 8, 0),
         ("qwen15", 32, None), ("qwen15", 160, 0), ("qwen2", 24, None), ("qwen3next", 16, 0),
         ("mixtral_8x7b", 1, None)]


def run_case(name, T, tc_min):
    import torch
    from any_precision_expert_pw_b200.device_layer import DeviceLayer

    cfg = CONFIGS[name] if name in CONFIGS else SCALED[name]
    L = make_layer(cfg, T)
    D = DeviceLayer(L)
    ref = olayer.moe_layer(L)
    dev = D.device
    idx = torch.from_numpy(np.ascontiguousarray(ref["idx"], np.int32)).to(dev)
    gate = torch.from_numpy(np.ascontiguousarray(ref["gate"], np.float32)).to(dev)
    n_y = D.T * D.H
    ybuf = torch.full((GUARD_WORDS + n_y + GUARD_WORDS,), Y_PATTERN, dtype=torch.int32,
                      device=dev)
    y = ybuf[GUARD_WORDS:GUARD_WORDS + n_y]
    wbuf = torch.full((D.ws_bytes + GUARD_BYTES,), WS_PATTERN, dtype=torch.uint8, device=dev)
    if tc_min is not None:
        B.check(B.pw_set_tc_min_tokens(tc_min))
    try:
        st = B.pw_moe_anyprec_forward(D.pt_dev.data_ptr(), 0, D.E, D.x.data_ptr(), D.T, D.H,
                                      D.I, D.k, idx.data_ptr(), gate.data_ptr(), y.data_ptr(),
                                      wbuf.data_ptr(), D.ws_bytes, D.stream)
        torch.cuda.synchronize()
    finally:
        B.check(B.pw_set_tc_min_tokens(4))
    dev_status = D.status()
    head = ybuf[:GUARD_WORDS].cpu().numpy()
    tail = ybuf[GUARD_WORDS + n_y:].cpu().numpy()
    wtail = wbuf[D.ws_bytes:].cpu().numpy()
    got = y.view(torch.float32).cpu().numpy().reshape(D.T, D.H)
    err, rms = ffn_err(got, ref["y"])
    res = {"case": f"{name}:T{T}:{'tc' if tc_min == 0 else 'auto'}", "status": st,
           "device_status": dev_status,
           "y_guards_ok": bool((head == Y_PATTERN).all() and (tail == Y_PATTERN).all()),
           "ws_guard_ok": bool((wtail == WS_PATTERN).all()),
           "err_over_rms": err / rms if rms > 0 else None}
    res["ok"] = (st == B.PW_OK and dev_status == B.PW_OK and res["y_guards_ok"] and
                 res["ws_guard_ok"] and rms > 0 and err <= FFN_RTOL_RMS * rms)
    return res


def main():
    want_debug = os.environ.get("PW_LIB_VARIANT") == "debug"
    version = B.pw_version()
    if ("debug" in version) != want_debug:
        print(json.dumps({"error": f"wrong library variant loaded: {version}"}))
        return 1
    print(json.dumps({"library": version, "path": B.LIB_PATH}))
    for name, T, tc_min in CASES:
        res = run_case(name, T, tc_min)
        print(json.dumps(res), flush=True)
        if not res["ok"]:
            return 1
    return 0


if __name__ == "__main__":
    sys.exit(main())
