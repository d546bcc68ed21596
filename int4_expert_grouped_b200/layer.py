"""One MoE layer held on the GPU: device buffers from torch, compute in the
C-ABI library.

``MoeLayer`` uploads the logical int4 weights, prepacks them once with
``moe_prepack_weights``, keeps the router weights and the workspace, and
exposes ``route``, ``forward`` and ``forward_host`` (the C entry points of
the same names).  Nothing here computes any part of the layer.
"""
from __future__ import annotations

import numpy as np
import torch

from . import Plan


def _dev(a: np.ndarray, device) -> torch.Tensor:
    """numpy -> device tensor with the same bytes (uint16 goes through int16)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(device)


def bf16_tensor(bits: np.ndarray, device) -> torch.Tensor:
    return _dev(bits, device).view(torch.bfloat16)


class MoeLayer:
    def __init__(self, T_max, d, E, k, f, group, gate, up, down, w_r, b_r=None,
                 device="cuda", keep_logical=False, flags=0):
        """gate/up/down: objects with .q (uint8 [E,N,K/2]), .scale, .bias
        (uint16 bf16 bits [E,N,K/group]); w_r float32 [d,E]; b_r float32 [E]."""
        self.device = torch.device(device)
        self.T_max, self.d, self.E, self.k, self.f, self.group = T_max, d, E, k, f, group
        self.plan = Plan(T_max, d, E, k, f, group, flags)
        info = self.plan.info
        logical = [tuple(_dev(getattr(p, n), self.device) for n in ("q", "scale", "bias"))
                   for p in (gate, up, down)]
        self.packed = torch.empty(info.packed_weight_bytes, dtype=torch.uint8, device=self.device)
        self.plan.prepack_weights(*logical, self.packed)
        self.logical = logical if keep_logical else None
        self.w_r = _dev(np.asarray(w_r, np.float32), self.device)
        self.b_r = None if b_r is None else _dev(np.asarray(b_r, np.float32), self.device)
        self.ws = torch.empty(info.workspace_bytes, dtype=torch.uint8, device=self.device)
        self._host_ws = None
        torch.cuda.synchronize(self.device)

    @classmethod
    def from_inputs(cls, inp, T_max=None, device="cuda", keep_logical=False, flags=0):
        s = inp.shape
        return cls(T_max or s.T, s.d, s.E, s.k, s.f, s.group, inp.gate, inp.up, inp.down,
                   inp.w_r, inp.b_r, device=device, keep_logical=keep_logical, flags=flags)

    def route_buffers(self, T):
        dev, k, E = self.device, self.k, self.E
        i32 = dict(dtype=torch.int32, device=dev)
        return {
            "topk_idx": torch.empty((max(T, 1), k), **i32),
            "topk_w": torch.empty((max(T, 1), k), dtype=torch.float32, device=dev),
            "counts": torch.empty(E, **i32),
            "offsets": torch.empty(E + 1, **i32),
            "sorted_assign": torch.empty(max(T * k, 1), **i32),
            "pos": torch.empty(max(T * k, 1), **i32),
            "block_offsets": torch.empty(E + 1, **i32),
            "block_map": torch.empty((self.plan.info.max_blocks, 3), **i32),
            "num_blocks": torch.empty(4, **i32),
        }

    def route(self, x: torch.Tensor, out=None, stream=None):
        T = x.shape[0]
        out = out or self.route_buffers(T)
        self.plan.route(T, x, self.w_r, self.b_r, out, self.ws, stream=stream)
        return out

    def forward(self, x: torch.Tensor, y: torch.Tensor | None = None, route_out=None, stream=None,
                events=None):
        T = x.shape[0]
        if y is None:
            y = torch.empty((max(T, 1), self.d), dtype=torch.bfloat16, device=self.device)
        self.plan.forward(T, x, self.w_r, self.b_r, self.packed, y, self.ws,
                          route_out=route_out, stream=stream, events=events)
        return y

    def host_workspace(self):
        if self._host_ws is None:
            self._host_ws = torch.empty(self.plan.info.host_workspace_bytes, dtype=torch.uint8,
                                        device=self.device)
        return self._host_ws

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, stream=None):
        """x_host, y_host: CPU bf16 tensors [T, d] (pinned for full speed)."""
        T = x_host.shape[0]
        self.plan.forward_host(T, x_host, self.w_r, self.b_r, self.packed, y_host,
                               self.host_workspace(), stream=stream)
        return y_host

    def read_status(self, clear=True):
        return self.plan.read_status(self.ws, clear=clear)
