"""Any-precision expert FFN and gate-weighted combine (oracle; test infrastructure only).

PagedWeight, "Composants Clés" 1 and 3: each (layer, expert, module) linear block is read at its
own committed bitwidth q from stacked bit-planes and a look-up table.  Dequantisation here is
W[r, c] = lut_q[r][top q bits of idx[r, c]], exact in float64 (fp16 -> float64 is exact).

The expert FFN (reading of "fused mixed-precision MoE kernel" for a gated MoE layer):
gate = W_gate x, up = W_up x (rows 0..I-1 and I..2I-1 of gate_up), h = SiLU(gate) * up with
SiLU(z) = z / (1 + e^-z), o = W_down h.  The layer output is y[t] = sum over slots, in slot
order, of gate[t, slot] * o[t, slot].  All in float64; rows are streamed so that no dense
float64 copy of a whole block is held.
"""
from __future__ import annotations

import numpy as np

from .bitplanes import child_index
from .group import group_by_expert
from .router import bf16_bits_to_f64


def silu(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def dequant_rows(idx_rows: np.ndarray, lut_q: np.ndarray, n: int, q: int) -> np.ndarray:
    """float64 [r, C]: lut_q[row][idx >> (n - q)] for each element of the given rows."""
    iq = child_index(idx_rows, n, q)
    return np.take_along_axis(np.asarray(lut_q, dtype=np.float64), iq, axis=1)


def block_matvec(idx: np.ndarray, lut_q: np.ndarray, n: int, q: int, X: np.ndarray,
                 row_chunk: int = 2048) -> np.ndarray:
    """W @ X for the dequantised block W [R, C] and X [C, Te] -> [R, Te], streaming rows."""
    R = idx.shape[0]
    out = np.empty((R, X.shape[1]), dtype=np.float64)
    for r0 in range(0, R, row_chunk):
        r1 = min(R, r0 + row_chunk)
        out[r0:r1] = dequant_rows(idx[r0:r1], lut_q[r0:r1], n, q) @ X
    return out


def expert_ffn(idx_gu, lut_gu_q, q_gu, idx_dn, lut_dn_q, q_dn, n, X):
    """X float64 [Te, H] -> expert output float64 [Te, H]."""
    I = idx_gu.shape[0] // 2
    GU = block_matvec(idx_gu, lut_gu_q, n, q_gu, X.T)       # [2I, Te]
    h = silu(GU[:I]) * GU[I:]                                # [I, Te]
    return block_matvec(idx_dn, lut_dn_q, n, q_dn, h).T      # [Te, H]


def moe_ffn(layer, idx, gate, q=None, experts_only=None):
    """Grouped FFN + combine for a SynthLayer; returns (y float64 [T, H], out float64 [T*k, H]).

    q overrides the layer's committed bitwidths ([E, 2]); experts_only restricts the work to
    the tokens whose assignments all fall in that set (used for sampled checks)."""
    idx = np.asarray(idx, dtype=np.int32)
    gate = np.asarray(gate, dtype=np.float32)
    T, k = idx.shape
    E, n = layer.cfg.E, layer.cfg.n
    qq = layer.q if q is None else np.asarray(q)
    X = bf16_bits_to_f64(layer.x_bf16)
    _, offsets, perm, active = group_by_expert(idx, E)
    out = np.zeros((T * k, layer.cfg.H), dtype=np.float64)
    for e in active:
        if experts_only is not None and int(e) not in experts_only:
            continue
        a = perm[offsets[e]:offsets[e + 1]]
        tokens = a // k
        qg, qd = int(qq[e, 0]), int(qq[e, 1])
        out[a] = expert_ffn(layer.idx[e][0], layer.lut[e][0][qg], qg,
                            layer.idx[e][1], layer.lut[e][1][qd], qd, n, X[tokens])
    y = np.zeros((T, layer.cfg.H), dtype=np.float64)
    for s in range(k):
        y += gate[:, s].astype(np.float64)[:, None] * out[np.arange(T) * k + s]
    return y, out
