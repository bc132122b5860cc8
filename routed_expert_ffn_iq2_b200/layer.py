"""Convenience owner of the device buffers one routed layer needs (grids,
slot table, expert pool, workspace, status word), built on the C ABI.
Torch provides the allocations and the stream; the library does the work."""

from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import numpy as np
import torch

from . import _native as N


class MoeLayer:
    def __init__(self, hidden: int, n_experts: int, max_ffn: int, max_tokens: int, top_k: int, grid_iq2, grid_iq1,
                 pool_bytes: int, device: str = "cuda", stream: Optional[torch.cuda.Stream] = None):
        self.hidden, self.n_experts, self.max_ffn = hidden, n_experts, max_ffn
        self.max_tokens, self.top_k = max_tokens, top_k
        self.device = torch.device(device)
        self.stream = stream if stream is not None else torch.cuda.current_stream(self.device)
        self.grids = torch.zeros(N.redlite_moe_grids_bytes(), dtype=torch.uint8, device=self.device)
        rc = N.redlite_moe_expand_grids(grid_iq2, grid_iq1, self.grids, self.stream)
        N._check(rc, "redlite_moe_expand_grids")
        # one spare slot past n_experts holds the shared expert's descriptor
        self.table_dev = torch.zeros((n_experts + 1) * ctypes.sizeof(N.redlite_moe_expert), dtype=torch.uint8,
                                     device=self.device)
        ws = N.redlite_moe_workspace_bytes(hidden, n_experts, max_tokens, top_k, max_ffn)
        self.workspace = torch.zeros(max(ws, 256), dtype=torch.uint8, device=self.device)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.pool = torch.empty(max(pool_bytes, 16), dtype=torch.uint8, device=self.device)
        self.pool_used = 0
        self.counters = N.redlite_moe_upload_counters()
        self.shared: Optional[N.redlite_moe_expert] = None
        self.table = N.redlite_moe_table(
            hidden, n_experts, max_ffn, max_tokens, 0, 0, self.table_dev.data_ptr(), self.grids.data_ptr(),
            self.workspace.data_ptr(), self.workspace.numel(), self.status.data_ptr(), self.stream.cuda_stream)
        N._check(N.redlite_moe_workspace_reset(self.table), "redlite_moe_workspace_reset")

    def upload(self, ids: Sequence[int], experts: Sequence) -> int:
        rc, end = N.redlite_moe_upload_experts(self.hidden, list(ids), list(experts), self.pool, self.pool_used,
                                               self.table_dev, self.n_experts + 1, self.counters, self.stream)
        if rc == N.REDLITE_OK:
            self.pool_used = end
            f = min(int(e.ffn) for e in experts) if len(experts) else 0
            self.table.min_ffn = f if self.table.min_ffn == 0 else min(self.table.min_ffn, f)
        return rc

    def set_shared(self, expert) -> int:
        if expert is None:
            self.shared = None
            return N.REDLITE_OK
        rc = self.upload([self.n_experts], [expert])
        if rc != N.REDLITE_OK:
            return rc
        raw = self.table_dev[self.n_experts * 32:(self.n_experts + 1) * 32].cpu().numpy().tobytes()
        self.shared = N.redlite_moe_expert.from_buffer_copy(raw)
        return rc

    def __call__(self, x: torch.Tensor, ids: torch.Tensor, weights: torch.Tensor,
                 out: Optional[torch.Tensor] = None, check: bool = True):
        T = x.shape[0]
        k = ids.shape[1] if ids.dim() == 2 else 1
        if out is None:
            out = torch.empty((T, self.hidden), dtype=torch.float32, device=self.device)
        rc = N.redlite_moe_layer(x, T, ids, weights, k, self.table, self.shared, out)
        if check:
            N._check(rc, "redlite_moe_layer")
        return out if check else (out, rc)

    def read_status(self) -> int:
        return int(self.status.item())

    def clear_status(self):
        self.status.zero_()

