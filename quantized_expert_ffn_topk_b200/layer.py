"""Device-memory owners over the C calls: one layer's resident arena and a
workspace. Allocation is torch's; all arithmetic happens in libmoeq.so."""
from __future__ import annotations

import torch

from . import (moe_combine_residual, moe_expert_bytes, moe_expert_ffn_q, moe_expert_layout, moe_layer_q,
               moe_pack_expert, moe_router_topk, moe_workspace_bytes, moe_workspace_init)

GATE, UP, DOWN = 0, 1, 2


class Workspace:
    """Caller-owned scratch for up to B tokens of a layer shape, zeroed once."""

    def __init__(self, B: int, K: int, H: int, I: int, E: int, device="cuda", stream=None):
        self.nbytes = moe_workspace_bytes(B, K, H, I, E)
        if self.nbytes == 0:
            raise ValueError("bad workspace shape")
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        moe_workspace_init(self.buf, self.nbytes, stream)

    def data_ptr(self) -> int:
        return self.buf.data_ptr()


class QuantLayer:
    """One MoE layer resident in HBM: E routed expert records, one shared
    record, the bf16 router matrix and an optional shared-gate vector."""

    def __init__(self, H: int, I: int, E: int, K: int, group: int, bits_routed: int = 4, bits_shared: int = 4,
                 shared_gate: bool = False, device="cuda"):
        self.H, self.I, self.E, self.K, self.group = H, I, E, K, group
        self.bits_routed, self.bits_shared = bits_routed, bits_shared
        self.rec_r = moe_expert_bytes(H, I, bits_routed, group)
        self.rec_s = moe_expert_bytes(H, I, bits_shared, group)
        if self.rec_r == 0 or self.rec_s == 0:
            raise ValueError("unsupported layer shape")
        self.lay_r = moe_expert_layout(H, I, bits_routed, group)
        self.lay_s = moe_expert_layout(H, I, bits_shared, group)
        self.experts = torch.empty(E * self.rec_r, dtype=torch.uint8, device=device)
        self.shared = torch.empty(self.rec_s, dtype=torch.uint8, device=device)
        self.router_w = torch.empty((E, H), dtype=torch.bfloat16, device=device)
        self.shared_gate_w = torch.empty(H, dtype=torch.bfloat16, device=device) if shared_gate else None
        self._struct = moe_layer_q(H, I, E, K, group, bits_routed, bits_shared, self.experts.data_ptr(),
                                   self.shared.data_ptr(), self.router_w.data_ptr(),
                                   self.shared_gate_w.data_ptr() if shared_gate else None)

    @property
    def struct(self) -> moe_layer_q:
        return self._struct

    def nbytes(self) -> int:
        n = self.experts.numel() + self.shared.numel() + self.router_w.numel() * 2
        return n + (self.shared_gate_w.numel() * 2 if self.shared_gate_w is not None else 0)

    def matrix_shape(self, matrix: int):
        return (self.I, self.H) if matrix in (GATE, UP) else (self.H, self.I)

    def record_ptr(self, expert: int) -> int:
        """Device address of expert `expert`'s record (expert == E: shared)."""
        if expert == self.E:
            return self.shared.data_ptr()
        return self.experts.data_ptr() + expert * self.rec_r

    def pack_expert(self, expert: int, gate, up, down, ws=None, stream=None) -> None:
        """Pack one expert (each matrix: device u8 codes, bf16 scale/bias) into its record."""
        bits = self.bits_shared if expert == self.E else self.bits_routed
        moe_pack_expert(gate, up, down, self.H, self.I, bits, self.group, self.record_ptr(expert), ws, stream)

    def fill(self, fill_matrix, ws=None, stream=None) -> None:
        """Build every record: fill_matrix(expert, matrix, codes_ptr, scale_ptr, bias_ptr)
        writes one matrix's u8 codes and bf16 scale/bias into scratch device
        buffers, which are then packed into the arena."""
        n = self.I * self.H
        dev = self.experts.device
        bufs = [(torch.empty(n, dtype=torch.uint8, device=dev), torch.empty(n // self.group, dtype=torch.bfloat16, device=dev),
                 torch.empty(n // self.group, dtype=torch.bfloat16, device=dev)) for _ in range(3)]
        for e in range(self.E + 1):
            for m in (GATE, UP, DOWN):
                c, s, b = bufs[m]
                fill_matrix(e, m, c.data_ptr(), s.data_ptr(), b.data_ptr())
            self.pack_expert(e, bufs[GATE], bufs[UP], bufs[DOWN], ws, stream)

    def forward(self, x, ws: Workspace, out: dict, resid_in=None, renorm=False, forced_idx=None, eps=None,
                stream=None) -> dict:
        """A1..A6 for B tokens through the three per-token calls.
        out holds preallocated idx [B,K] i32, w [B,K] f32, y [B,K+1,H] f32,
        resid [B,H] f32, optional logits [B,E] f32 and xnorm [B,H] bf16."""
        B = x.shape[0]
        moe_router_topk(x, self.router_w, B, self.H, self.E, self.K, renorm, forced_idx, out["idx"], out["w"],
                        out.get("logits"), ws.buf, ws.nbytes, stream)
        moe_expert_ffn_q(self._struct, x, B, out["idx"], out["y"], ws.buf, ws.nbytes, stream)
        moe_combine_residual(self._struct, out["y"], out["w"], x, resid_in, B, out["resid"],
                             out.get("xnorm") if eps is not None else None, eps if eps is not None else 0.0, stream)
        return out

    def alloc_outputs(self, B: int, logits=True, xnorm=True) -> dict:
        dev = self.experts.device
        out = dict(idx=torch.empty((B, self.K), dtype=torch.int32, device=dev),
                   w=torch.empty((B, self.K), dtype=torch.float32, device=dev),
                   y=torch.empty((B, self.K + 1, self.H), dtype=torch.float32, device=dev),
                   resid=torch.empty((B, self.H), dtype=torch.float32, device=dev))
        if logits:
            out["logits"] = torch.empty((B, self.E), dtype=torch.float32, device=dev)
        if xnorm:
            out["xnorm"] = torch.empty((B, self.H), dtype=torch.bfloat16, device=dev)
        return out
