"""Shared helpers of the GPU parity tests (comparison rules and sizes)."""
import numpy as np

from any_precision_expert_pw_b200 import binding as B
from any_precision_expert_pw_b200.inputs import CONFIGS

FFN_RTOL_RMS = 2e-3        # max |y_gpu - y_ref| <= 2e-3 * rms(y_ref)
GATE_ATOL = 1e-6           # routing gates (fp32 vs float64, rounded once on both sides)

# scaled-down shapes: several tiles, ragged column tails (H or I not a multiple of 512)
SCALED = {
    "tiny": CONFIGS["tiny"],
    "qwen15": CONFIGS["qwen15_moe_a2.7b"].scaled(H=640, I=384),
    "mixtral": CONFIGS["mixtral_8x7b"].scaled(H=1152, I=1408),
    "qwen3next": CONFIGS["qwen3_next_80b_a3b"].scaled(H=384, I=256),
    "qwen2": CONFIGS["qwen2_57b_a14b"].scaled(H=896, I=640),
}


def ffn_err(y_gpu, y_ref):
    y_ref = np.asarray(y_ref, np.float64)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    err = float(np.max(np.abs(np.asarray(y_gpu, np.float64) - y_ref)))
    return err, rms


def assert_ffn_close(y_gpu, y_ref, what=""):
    err, rms = ffn_err(y_gpu, y_ref)
    assert rms > 0, what
    assert err <= FFN_RTOL_RMS * rms, f"{what}: max err {err:.3e} > {FFN_RTOL_RMS} * rms {rms:.3e}"
    return err / rms


def tiled_reference(planes, layout):
    """The tiled arrangement of [n][rows][words] bit-planes, built with array reshapes: row
    tiles of 32 (gate_up: 16 gate rows then the 16 matching up rows), stages of 16 words, and
    inside a stage [plane][word][row]."""
    n, R, W = planes.shape
    if layout == B.PW_LAYOUT_TILED_GATE_UP:
        half = R // 2
        order = np.concatenate([np.r_[16 * t:16 * t + 16, half + 16 * t:half + 16 * t + 16]
                                for t in range(half // 16)])
    else:
        order = np.arange(R)
    tiles = planes[:, order, :].reshape(n, R // 32, 32, W)
    out = []
    for t in range(R // 32):
        for s0 in range(0, W, 16):
            blk = tiles[:, t, :, s0:s0 + 16]                      # [n][32 rows][ws words]
            out.append(blk.transpose(0, 2, 1).reshape(-1))        # [n][ws][32]
    return np.concatenate(out)
