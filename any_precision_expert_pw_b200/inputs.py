"""Seeded synthetic MoE decode layers (the inputs both the CUDA path and the oracle consume).

This module holds the data recipe only: random draws, the rounding of those draws to their
storage types, and the construction of the nested per-row look-up tables that define the
synthetic Any-Precision weights.  It computes nothing the decode layer computes (no routing,
no packing, no decoding, no FFN); the CUDA library and the CPU oracle both start from what
it returns.

Recipe (one MoE layer, layer 0, per case):

* seeds: ``numpy.random.SeedSequence([cfg_id, T, stream] + shape)`` where ``shape`` is empty for
  the named shapes and ``[H, E, I]`` for a scaled-down variant; streams are 0 = per-block
  bitwidth q, 1 = parent indices, 2 = parent LUT draws, 3 = router weight W_r, 4 = Zipf
  permutation, 5 = activations x, 6 = resident set.
* parent indices: iid uniform over [0, 2^n) per (row, column) of each linear block, uint8.
* parent LUT per row: 2^n draws of N(0, 0.02), rounded to fp16 (round-to-nearest-even), sorted.
* child LUT for b < n: entry j is the fp16 rounding of the float64 mean of the parent entries
  whose top b bits equal j (entries j*2^(n-b) ... (j+1)*2^(n-b)-1), so each b-bit table is
  "nested by top bits" in the parent and stays sorted.  Every b in [min_bits, n] is stored, so a
  change of committed bitwidth needs no new data.
* router: W_r ~ N(0, 0.02) fp32 [E, H]; bias zero except a Zipf(s) skew where
  bias_e = ln(rho_pi(e)), rho_j = j^-s / sum_i i^-s, pi a seeded permutation of 1..E.
* activations: x ~ N(0, 1) drawn in float64, rounded to fp32 then to bf16 (both RNE).
* residency: exactly floor(frac * E) experts, drawn without replacement.
* block order (for the index and LUT streams): expert 0 gate_up, expert 0 down, expert 1 ...
  gate_up is [2I, H] with gate rows 0..I-1 and up rows I..2I-1; down is [H, I].

The five named shapes follow the models the pages evaluate (PagedWeight, "Principales
Contributions" 4; the substitution page, "Méthodologie"; LYNX, section 1); none of those
models' weights are used or needed.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

MOD_GATE_UP = 0
MOD_DOWN = 1
MIN_BITS = 3

POLICY_NONE = -1      # no residency rule and no remap (plain top-k routing)
POLICY_FETCH_ALL = 0
POLICY_THRESHOLD = 1
POLICY_FIRST_CHOICE = 2
POLICY_REMAP = 3
POLICY_AFFINITY = 4   # LYNX AffinityBinning remap (bins from k/N), in place of POLICY_REMAP


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    cfg_id: int
    H: int
    E: int
    I: int
    k: int
    renorm: bool
    n: int                                  # parent bits
    q_values: Tuple[int, ...]
    q_weights: Optional[Tuple[float, ...]]  # None = uniform
    T_sweep: Tuple[int, ...]
    zipf_s: Optional[float] = None
    resident_frac: Optional[float] = None
    policy: int = POLICY_NONE
    threshold: float = 0.15
    critical_n: int = 32

    def scaled(self, H: int, I: int, E: Optional[int] = None) -> "LayerConfig":
        """Same routing/bitwidth recipe at a smaller H, I (and optionally E)."""
        return dataclasses.replace(self, name=f"{self.name}@H{H}I{I}E{E or self.E}", H=H, I=I,
                                   E=E or self.E)


CONFIGS: Dict[str, LayerConfig] = {
    "tiny": LayerConfig("tiny", 1, H=256, E=8, I=512, k=2, renorm=False, n=4,
                        q_values=(3, 4), q_weights=None, T_sweep=(4,)),
    "qwen15_moe_a2.7b": LayerConfig("qwen15_moe_a2.7b", 2, H=2048, E=60, I=1408, k=4, renorm=True,
                                    n=8, q_values=(3, 4, 5, 6, 7, 8),
                                    q_weights=(1, 3, 3, 1, 1, 1), T_sweep=(32,)),
    "mixtral_8x7b": LayerConfig("mixtral_8x7b", 3, H=4096, E=8, I=14336, k=2, renorm=True, n=8,
                                q_values=(3, 4, 5, 6, 7, 8), q_weights=None,
                                T_sweep=(1, 8, 64, 256), zipf_s=1.2),
    "qwen3_next_80b_a3b": LayerConfig("qwen3_next_80b_a3b", 4, H=2048, E=512, I=512, k=10,
                                      renorm=True, n=4, q_values=(3, 4), q_weights=None,
                                      T_sweep=(1, 16), resident_frac=0.25,
                                      policy=POLICY_THRESHOLD, threshold=0.15),
    "qwen2_57b_a14b": LayerConfig("qwen2_57b_a14b", 5, H=3584, E=64, I=2560, k=8, renorm=False,
                                  n=8, q_values=(3, 4, 5, 6, 7, 8), q_weights=None,
                                  T_sweep=(8, 32, 64), policy=POLICY_REMAP, critical_n=32),
}


@dataclasses.dataclass
class SynthLayer:
    cfg: LayerConfig
    T: int
    q: np.ndarray                       # uint8 [E, 2] committed bitwidth per (expert, module)
    idx: List[List[np.ndarray]]         # idx[e][m] uint8 [R, C] parent indices
    lut: List[List[Dict[int, np.ndarray]]]  # lut[e][m][b] float16 [R, 2^b], b in [MIN_BITS, n]
    Wr: np.ndarray                      # float32 [E, H]
    bias: np.ndarray                    # float32 [E]
    x_bf16: np.ndarray                  # uint16 [T, H] (bf16 bit patterns)
    resident: Optional[np.ndarray]      # uint8 [E] or None

    @property
    def H(self) -> int:
        return self.cfg.H

    @property
    def E(self) -> int:
        return self.cfg.E

    @property
    def I(self) -> int:
        return self.cfg.I

    def block_shape(self, m: int) -> Tuple[int, int]:
        return block_shape(self.cfg, m)


def block_shape(cfg: LayerConfig, m: int) -> Tuple[int, int]:
    return (2 * cfg.I, cfg.H) if m == MOD_GATE_UP else (cfg.H, cfg.I)


def _rng(cfg: LayerConfig, T: int, stream: int) -> np.random.Generator:
    key = [cfg.cfg_id, T, stream]
    base = CONFIGS.get(cfg.name)
    if base is None or (base.H, base.E, base.I) != (cfg.H, cfg.E, cfg.I):
        key += [cfg.H, cfg.E, cfg.I]
    return np.random.default_rng(np.random.SeedSequence(key))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round-to-nearest-even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def nested_luts(parent: np.ndarray, n: int, min_bits: int = MIN_BITS) -> Dict[int, np.ndarray]:
    """Per-row child tables nested by top bits in a sorted fp16 parent table [R, 2^n]."""
    out = {n: parent}
    p64 = parent.astype(np.float64)
    R = parent.shape[0]
    for b in range(min_bits, n):
        g = 1 << (n - b)
        out[b] = p64.reshape(R, 1 << b, g).mean(axis=2).astype(np.float16)
    return out


def draw_bitwidths(cfg: LayerConfig, T: int) -> np.ndarray:
    rng = _rng(cfg, T, 0)
    p = None
    if cfg.q_weights is not None:
        w = np.asarray(cfg.q_weights, dtype=np.float64)
        p = w / w.sum()
    q = rng.choice(np.asarray(cfg.q_values), size=2 * cfg.E, p=p)
    return q.reshape(cfg.E, 2).astype(np.uint8)


def make_layer(cfg: LayerConfig, T: int, with_weights: bool = True) -> SynthLayer:
    """Build one seeded synthetic layer; with_weights=False skips the (large) index/LUT draws."""
    E, H, n = cfg.E, cfg.H, cfg.n
    q = draw_bitwidths(cfg, T)

    idx: List[List[np.ndarray]] = []
    lut: List[List[Dict[int, np.ndarray]]] = []
    if with_weights:
        ri, rl = _rng(cfg, T, 1), _rng(cfg, T, 2)
        for e in range(E):
            idx_e, lut_e = [], []
            for m in (MOD_GATE_UP, MOD_DOWN):
                R, C = block_shape(cfg, m)
                idx_e.append(ri.integers(0, 1 << n, size=(R, C), dtype=np.uint8))
                parent = np.sort(rl.normal(0.0, 0.02, size=(R, 1 << n)).astype(np.float16), axis=1)
                lut_e.append(nested_luts(parent, n))
            idx.append(idx_e)
            lut.append(lut_e)

    Wr = _rng(cfg, T, 3).normal(0.0, 0.02, size=(E, H)).astype(np.float32)
    bias = np.zeros(E, dtype=np.float32)
    if cfg.zipf_s is not None:
        perm = _rng(cfg, T, 4).permutation(E) + 1
        j = np.arange(1, E + 1, dtype=np.float64)
        rho = j ** (-cfg.zipf_s)
        rho /= rho.sum()
        bias = np.log(rho[perm - 1]).astype(np.float32)
    x = _rng(cfg, T, 5).standard_normal((T, H)).astype(np.float32)
    x_bf16 = f32_to_bf16_bits(x)
    resident = None
    if cfg.resident_frac is not None:
        nres = int(math.floor(cfg.resident_frac * E))
        resident = np.zeros(E, dtype=np.uint8)
        resident[_rng(cfg, T, 6).choice(E, size=nres, replace=False)] = 1
    return SynthLayer(cfg, T, q, idx, lut, Wr, bias, x_bf16, resident)


def random_router_inputs(T: int, E: int, H: int, seed: int, zipf_s: Optional[float] = None):
    """Router-only inputs (x bf16 bits, W_r, bias) for routing tests at arbitrary shapes."""
    rng = np.random.default_rng(np.random.SeedSequence([9001, T, E, H, seed]))
    Wr = rng.normal(0.0, 0.02, size=(E, H)).astype(np.float32)
    x_bf16 = f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    bias = np.zeros(E, dtype=np.float32)
    if zipf_s is not None:
        perm = rng.permutation(E) + 1
        j = np.arange(1, E + 1, dtype=np.float64)
        rho = j ** (-zipf_s)
        rho /= rho.sum()
        bias = np.log(rho[perm - 1]).astype(np.float32)
    return x_bf16, Wr, bias


def random_indices(R: int, C: int, n: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(np.random.SeedSequence([9002, R, C, n, seed]))
    return rng.integers(0, 1 << n, size=(R, C), dtype=np.uint8)


def logit_stream(E: int, T: int, steps: int, seed: int, topic_len: int = 16,
                 topic_scale: float = 2.0) -> np.ndarray:
    """Router logits for a run of decode steps [steps][T][E] (fp32): standard normal noise plus
    a per-topic bias that changes every `topic_len` steps (a random permutation of a Zipf(1.2)
    log-profile times `topic_scale`), standing in for a real model's routing stream."""
    rng = np.random.default_rng(np.random.SeedSequence([7, E, T, steps, seed]))
    prof = np.log(np.arange(1, E + 1, dtype=np.float64) ** -1.2)
    prof -= prof.mean()
    out = np.empty((steps, T, E), dtype=np.float32)
    bias = None
    for s in range(steps):
        if s % topic_len == 0:
            bias = topic_scale * prof[rng.permutation(E)] / max(prof.std(), 1e-12)
        out[s] = (rng.standard_normal((T, E)) + bias).astype(np.float32)
    return out


def synthetic_damage(num_blocks: int, seed: int, hot_frac: float = 0.1,
                     hot_mult: float = 4.0) -> np.ndarray:
    """Per-block damage scores [num_blocks][9] (float64) for the bitwidth planner: a seeded
    log-normal sensitivity per block, times a multiplier for a seeded set of hot blocks, times
    4^-q (one more bit quarters the squared quantisation error); column q, q = 0..8."""
    rng = np.random.default_rng(np.random.SeedSequence([13, num_blocks, seed]))
    sens = rng.lognormal(mean=0.0, sigma=1.0, size=num_blocks)
    hot = rng.random(num_blocks) < hot_frac
    sens = sens * np.where(hot, hot_mult, 1.0)
    q = np.arange(9, dtype=np.float64)
    return sens[:, None] * np.power(4.0, -q)[None, :]
