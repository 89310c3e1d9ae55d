"""Device-resident decode layer: marshals a synthetic layer into libpw's buffers and calls it.

PyTorch is used only to allocate device memory and to name the stream; every step of the
layer (packing, routing, substitution or remap, grouping, the any-precision FFN and the
combine) runs in libpw's kernels.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import numpy as np

from . import binding as B
from .inputs import (MIN_BITS, MOD_DOWN, MOD_GATE_UP, POLICY_AFFINITY, POLICY_NONE, POLICY_REMAP,
                     SynthLayer)


def _torch():
    import torch
    return torch


def _dev_tensor(arr: np.ndarray, device):
    torch = _torch()
    return torch.from_numpy(np.ascontiguousarray(arr)).to(device)


def _bytes_tensor(obj: ctypes.Structure | ctypes.Array, device):
    torch = _torch()
    raw = bytearray(bytes(obj))
    return torch.frombuffer(raw, dtype=torch.uint8).to(device)


class DeviceLayer:
    """One MoE layer on one GPU: Weight Page Table (bit-planes + LUTs per block), router,
    activations, outputs and workspace, all in device memory owned by this object."""

    def __init__(self, L: SynthLayer, device: str = "cuda", pack_on_gpu: bool = True):
        torch = _torch()
        self.L = L
        cfg = L.cfg
        self.cfg = cfg
        self.device = torch.device(device)
        self.T, self.E, self.H, self.I, self.k = L.T, cfg.E, cfg.H, cfg.I, cfg.k
        self.stream = torch.cuda.current_stream(self.device).cuda_stream
        n = cfg.n
        self.num_blocks = 2 * cfg.E
        self.blocks_host = (B.pw_block * self.num_blocks)()
        self._keep = []
        self.planes = {}  # (expert, module) -> device plane buffer (tiled, all n planes)
        for e in range(cfg.E):
            for m in (MOD_GATE_UP, MOD_DOWN):
                R, C = L.block_shape(m)
                layout = B.PW_LAYOUT_TILED_GATE_UP if m == MOD_GATE_UP else B.PW_LAYOUT_TILED_DOWN
                planes = torch.empty((n * R * (C // 32),), dtype=torch.int32, device=self.device)
                idx_d = _dev_tensor(L.idx[e][m], self.device)
                B.check(B.pw_pack_bitplanes(idx_d.data_ptr(), R, C, n, layout, planes.data_ptr(),
                                            self.stream), "pw_pack_bitplanes")
                del idx_d
                parts = [L.lut[e][m][b].view(np.int16).reshape(-1) for b in range(MIN_BITS, n + 1)]
                lut_d = _dev_tensor(np.concatenate(parts), self.device)
                blk = self.blocks_host[e * 2 + m]
                blk.rows, blk.cols = R, C
                blk.parent_bits, blk.min_bits = n, MIN_BITS
                q = int(L.q[e, m])
                blk.desired_bits = blk.committed_bits = q
                blk.state = B.PW_PAGE_GPU
                blk.layout = layout
                blk.planes = planes.data_ptr()
                off = 0
                for b in range(MIN_BITS, n + 1):
                    blk.lut[b] = lut_d.data_ptr() + 2 * off
                    off += R * (1 << b)
                B.check(B.pw_block_prepare(blk), "pw_block_prepare")
                self._keep += [planes, lut_d]
                self.planes[(e, m)] = planes
        self.blocks_dev = _bytes_tensor(self.blocks_host, self.device)
        self.pt_host = B.pw_page_table(1, cfg.E, self.blocks_dev.data_ptr())
        self.pt_dev = _bytes_tensor(self.pt_host, self.device)

        self.Wr = _dev_tensor(L.Wr, self.device)
        self.bias = _dev_tensor(L.bias, self.device)
        self.x = _dev_tensor(L.x_bf16.view(np.int16), self.device)
        self.resident = (_dev_tensor(L.resident, self.device) if L.resident is not None else None)
        T, E, k, H = self.T, self.E, self.k, self.H
        f32, i32, u8 = torch.float32, torch.int32, torch.uint8
        self.logits = torch.empty((T, E), dtype=f32, device=self.device)
        self.idx = torch.empty((T, k), dtype=i32, device=self.device)
        self.gate = torch.empty((T, k), dtype=f32, device=self.device)
        self.action = torch.empty((T, k), dtype=u8, device=self.device)
        self.mass = torch.empty((T,), dtype=f32, device=self.device)
        self.critical = torch.empty((E,), dtype=u8, device=self.device)
        self.unique = torch.zeros((2,), dtype=i32, device=self.device)  # distinct experts
                                                                        # before / after a remap
        self.y = torch.empty((T, H), dtype=f32, device=self.device)
        self.ws_bytes = B.pw_moe_workspace_bytes(T, k, E, H, self.I)
        self.workspace = torch.empty((self.ws_bytes,), dtype=u8, device=self.device)
        self.route_cfg = B.pw_route_cfg(k=k, renorm=int(cfg.renorm),
                                        policy=max(cfg.policy, 0) if cfg.policy < POLICY_REMAP else 0,
                                        threshold=cfg.threshold, critical_n=cfg.critical_n)

    # ------------------------------------------------------------------ steps
    def route(self, x_ptr: Optional[int] = None) -> None:
        """Router + top-k + the layer's assignment rewrite (substitution or remap)."""
        x = self.x.data_ptr() if x_ptr is None else x_ptr
        B.check(B.pw_route_topk(x, self.Wr.data_ptr(), self.bias.data_ptr(), self.T, self.H,
                                self.E, self.route_cfg, self.logits.data_ptr(),
                                self.idx.data_ptr(), self.gate.data_ptr(), self.stream),
                "pw_route_topk")
        pol = self.cfg.policy
        if pol == POLICY_AFFINITY:
            acfg = B.pw_affinity_cfg()
            B.check(B.pw_affinity_default(self.E, self.k, acfg), "pw_affinity_default")
            B.check(B.pw_affinity_remap(self.logits.data_ptr(), self.idx.data_ptr(),
                                        self.gate.data_ptr(), self.T, self.E, self.route_cfg,
                                        acfg, self.critical.data_ptr(), 0,
                                        self.unique.data_ptr(), self.stream),
                    "pw_affinity_remap")
        elif pol == POLICY_REMAP:
            B.check(B.pw_remap(self.logits.data_ptr(), self.idx.data_ptr(), self.gate.data_ptr(),
                               self.T, self.E, self.route_cfg, self.critical.data_ptr(),
                               self.unique.data_ptr(), self.stream), "pw_remap")
        elif pol != POLICY_NONE:
            B.check(B.pw_substitute(self.logits.data_ptr(), self.idx.data_ptr(),
                                    self.gate.data_ptr(), self.resident.data_ptr(), self.T,
                                    self.E, self.route_cfg, self.action.data_ptr(),
                                    self.mass.data_ptr(), self.stream), "pw_substitute")

    def ffn(self, x_ptr: Optional[int] = None, idx_ptr: Optional[int] = None,
            gate_ptr: Optional[int] = None, y_ptr: Optional[int] = None) -> None:
        """Grouped any-precision FFN + combine on the current (or given) assignments."""
        B.check(B.pw_moe_anyprec_forward(
            self.pt_dev.data_ptr(), 0, self.E,
            self.x.data_ptr() if x_ptr is None else x_ptr, self.T, self.H, self.I, self.k,
            self.idx.data_ptr() if idx_ptr is None else idx_ptr,
            self.gate.data_ptr() if gate_ptr is None else gate_ptr,
            self.y.data_ptr() if y_ptr is None else y_ptr,
            self.workspace.data_ptr(), self.ws_bytes, self.stream), "pw_moe_anyprec_forward")

    def forward(self, x_ptr: Optional[int] = None) -> None:
        self.route(x_ptr)
        self.ffn(x_ptr)

    def commit(self, block_ids, q) -> None:
        """Commit bitwidths (stream-ordered) for the given block ids."""
        torch = _torch()
        ids = torch.as_tensor(np.asarray(block_ids, np.int32), device=self.device)
        qq = torch.as_tensor(np.asarray(q, np.uint8), device=self.device)
        B.check(B.pw_commit_bits(self.pt_dev.data_ptr(), self.num_blocks, ids.data_ptr(),
                                 qq.data_ptr(), len(ids), self.stream), "pw_commit_bits")
        self._keep.append((ids, qq))

    def status(self) -> int:
        return B.pw_get_status(self.stream)

    def committed_bits(self) -> np.ndarray:
        """[E, 2] committed bitwidths as stored in the device page table."""
        raw = self.blocks_dev.view(-1, 256)[:, 11].cpu().numpy()
        return raw.reshape(self.E, 2)

    def page_update(self, updates) -> None:
        """Apply pw_page_update_t edits (a list of dicts: block, state, stored_bits,
        committed_bits, planes) to the device table, stream-ordered."""
        torch = _torch()
        arr = (B.pw_page_update_t * len(updates))()
        for i, u in enumerate(updates):
            arr[i].block = u["block"]
            arr[i].state = u.get("state", -1) + 1
            arr[i].stored_bits = u.get("stored_bits", 0)
            arr[i].committed_bits = u.get("committed_bits", 0)
            arr[i].planes = u.get("planes", None)
        d = _bytes_tensor(arr, self.device)
        B.check(B.pw_page_update(self.pt_dev.data_ptr(), self.num_blocks, d.data_ptr(),
                                 len(updates), self.stream), "pw_page_update")
        self._keep.append(d)

    def set_state(self, e: int, m: int, state: int) -> None:
        """Change a block's page state in the device table (host-side test hook)."""
        self.blocks_dev.view(-1, 256)[e * 2 + m, 12] = state
