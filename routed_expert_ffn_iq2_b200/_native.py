"""ctypes binding of libredlite_moe.so: the C ABI of include/redlite_moe.h
with the same names.  Argument marshalling only -- torch supplies device
memory and the current stream; every step of the layer runs in the
library's CUDA kernels.  There is no fallback: if the library is missing
or fails to load, every call raises."""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libredlite_moe.so")

REDLITE_Q_IQ2XS_STYLE = 1
REDLITE_Q_IQ1M_STYLE = 2
REDLITE_Q_Q8_0_STYLE = 3
REDLITE_Q_Q4_K_STYLE = 4
REDLITE_OK = 0
REDLITE_EINVAL = -1
REDLITE_EUNSUPPORTED = -2
REDLITE_ENOMEM = -3
REDLITE_ECUDA = -4
REDLITE_EAGAIN = -5
REDLITE_STATUS_BAD_ID = 1
REDLITE_STATUS_BAD_EXPERT = 2
REDLITE_STATUS_TIMEOUT = 4

_c_void_p = ctypes.c_void_p


class redlite_moe_expert(ctypes.Structure):
    _fields_ = [("qtype", ctypes.c_int32), ("ffn", ctypes.c_int32), ("gate", _c_void_p), ("up", _c_void_p),
                ("down", _c_void_p)]


class redlite_moe_table(ctypes.Structure):
    _fields_ = [
        ("hidden", ctypes.c_int32), ("n_experts", ctypes.c_int32), ("max_ffn", ctypes.c_int32),
        ("max_tokens", ctypes.c_int32), ("min_ffn", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("experts", _c_void_p), ("grids", _c_void_p), ("workspace", _c_void_p),
        ("workspace_bytes", ctypes.c_size_t), ("status", _c_void_p), ("stream", _c_void_p),
    ]


class redlite_moe_pool_counters(ctypes.Structure):
    _fields_ = [("loads", ctypes.c_int64), ("hits", ctypes.c_int64), ("evictions", ctypes.c_int64),
                ("copies", ctypes.c_int64), ("bytes", ctypes.c_int64)]


class redlite_moe_upload_counters(ctypes.Structure):
    _fields_ = [("loads", ctypes.c_int64), ("copies", ctypes.c_int64), ("bytes", ctypes.c_int64)]


EXPORTS = {
    "redlite_moe_grids_bytes": (ctypes.c_size_t, []),
    "redlite_moe_expand_grids": (ctypes.c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p]),
    "redlite_moe_matrix_bytes": (ctypes.c_size_t, [ctypes.c_int32, ctypes.c_int64, ctypes.c_int64]),
    "redlite_moe_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int32] * 5),
    "redlite_moe_workspace_reset": (ctypes.c_int, [ctypes.POINTER(redlite_moe_table)]),
    "redlite_moe_layer": (ctypes.c_int, [_c_void_p, ctypes.c_int32, _c_void_p, _c_void_p, ctypes.c_int32,
                                         ctypes.POINTER(redlite_moe_table), ctypes.POINTER(redlite_moe_expert),
                                         _c_void_p]),
    "redlite_moe_layer_noalloc": (ctypes.c_int, [_c_void_p, ctypes.c_int32, _c_void_p, _c_void_p, ctypes.c_int32,
                                                 ctypes.POINTER(redlite_moe_table),
                                                 ctypes.POINTER(redlite_moe_expert), _c_void_p]),
    "redlite_moe_layer_host": (ctypes.c_int, [_c_void_p, _c_void_p, ctypes.c_int32, ctypes.c_int32,
                                              ctypes.POINTER(redlite_moe_table), ctypes.POINTER(redlite_moe_expert),
                                              _c_void_p, _c_void_p]),
    "redlite_moe_host_input_bytes": (ctypes.c_size_t, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]),
    "redlite_moe_route_topk": (ctypes.c_int, [_c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _c_void_p,
                                              _c_void_p, _c_void_p]),
    "redlite_moe_block_scratch_bytes": (ctypes.c_size_t, [ctypes.c_int32] * 4),
    "redlite_moe_block": (ctypes.c_int, [_c_void_p, ctypes.c_int32, _c_void_p, ctypes.c_float, _c_void_p,
                                         ctypes.c_int32, ctypes.POINTER(redlite_moe_table),
                                         ctypes.POINTER(redlite_moe_expert), _c_void_p, _c_void_p, ctypes.c_size_t]),
    "redlite_moe_pool_create": (_c_void_p, [ctypes.c_int32, ctypes.c_int32]),
    "redlite_moe_pool_destroy": (None, [_c_void_p]),
    "redlite_moe_pool_plan": (ctypes.c_int, [_c_void_p, _c_void_p, ctypes.c_int32, _c_void_p, _c_void_p, _c_void_p,
                                             ctypes.POINTER(ctypes.c_int64)]),
    "redlite_moe_pool_complete": (ctypes.c_int, [_c_void_p, ctypes.c_int64]),
    "redlite_moe_pool_release": (ctypes.c_int, [_c_void_p, ctypes.c_int64, _c_void_p]),
    "redlite_moe_pool_slot_of": (ctypes.c_int32, [_c_void_p, ctypes.c_int32]),
    "redlite_moe_pool_pins": (ctypes.c_int32, [_c_void_p, ctypes.c_int32]),
    "redlite_moe_pool_acquire": (ctypes.c_int, [_c_void_p, _c_void_p, ctypes.c_int32, _c_void_p, ctypes.c_int32,
                                                _c_void_p, ctypes.c_size_t, _c_void_p, _c_void_p, _c_void_p,
                                                ctypes.POINTER(redlite_moe_pool_counters),
                                                ctypes.POINTER(ctypes.c_int64)]),
    "redlite_proj_matrix_bytes": (ctypes.c_size_t, [ctypes.c_int32, ctypes.c_int64, ctypes.c_int64]),
    "redlite_proj_gemv": (ctypes.c_int, [ctypes.c_int32, _c_void_p, ctypes.c_int64, ctypes.c_int64, _c_void_p,
                                         ctypes.c_int32, _c_void_p, _c_void_p]),
    "redlite_moe_pack_matrix": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int64, ctypes.c_int64, _c_void_p,
                                               _c_void_p]),
    "redlite_moe_dequant": (ctypes.c_int, [ctypes.c_int32, _c_void_p, ctypes.c_int64, ctypes.c_int64, _c_void_p,
                                           _c_void_p, _c_void_p, _c_void_p]),
    "redlite_moe_upload_experts": (ctypes.c_int, [ctypes.c_int32, _c_void_p, _c_void_p, ctypes.c_int32, _c_void_p,
                                                  ctypes.c_size_t, ctypes.c_size_t, _c_void_p, ctypes.c_int32,
                                                  _c_void_p, ctypes.POINTER(redlite_moe_upload_counters),
                                                  ctypes.POINTER(ctypes.c_size_t)]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libredlite_moe.so (raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run routed_expert_ffn_iq2_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in EXPORTS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream: Optional[torch.cuda.Stream]):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int, what: str):
    if rc != REDLITE_OK:
        raise RuntimeError(f"{what} failed with code {rc}")


# ---------------------------------------------------------------- same-named calls


def redlite_moe_grids_bytes() -> int:
    return int(lib().redlite_moe_grids_bytes())


def redlite_moe_matrix_bytes(qtype: int, rows: int, k: int) -> int:
    return int(lib().redlite_moe_matrix_bytes(qtype, rows, k))


def redlite_moe_workspace_bytes(hidden: int, n_experts: int, max_tokens: int, top_k: int, max_ffn: int) -> int:
    return int(lib().redlite_moe_workspace_bytes(hidden, n_experts, max_tokens, top_k, max_ffn))


def redlite_moe_expand_grids(iq2_compact, iq1_compact, grids: torch.Tensor, stream=None) -> int:
    """iq2_compact / iq1_compact: host uint16 numpy arrays [512] / [2048]."""
    import numpy as np

    a = np.ascontiguousarray(iq2_compact, dtype=np.uint16)
    b = np.ascontiguousarray(iq1_compact, dtype=np.uint16)
    if a.size != 512 or b.size != 2048:
        return REDLITE_EINVAL
    return lib().redlite_moe_expand_grids(a.ctypes.data_as(_c_void_p), b.ctypes.data_as(_c_void_p), _ptr(grids),
                                          _stream_handle(stream))


def redlite_moe_dequant(qtype: int, packed: torch.Tensor, rows: int, k: int, grids: torch.Tensor,
                        out_f32: Optional[torch.Tensor], out_bf16: Optional[torch.Tensor], stream=None) -> int:
    return lib().redlite_moe_dequant(qtype, _ptr(packed), rows, k, _ptr(grids), _ptr(out_f32), _ptr(out_bf16),
                                     _stream_handle(stream))


def redlite_moe_pack_matrix(qtype: int, rows: int, k: int, src):
    """Interchange -> resident layout on the host (numpy uint8 in, numpy uint8 out)."""
    import numpy as np

    a = np.ascontiguousarray(src, dtype=np.uint8)
    out = np.zeros_like(a)
    rc = lib().redlite_moe_pack_matrix(qtype, rows, k, a.ctypes.data_as(_c_void_p), out.ctypes.data_as(_c_void_p))
    _check(rc, "redlite_moe_pack_matrix")
    return out


def redlite_moe_workspace_reset(table: redlite_moe_table) -> int:
    return lib().redlite_moe_workspace_reset(ctypes.byref(table))


def redlite_moe_layer(x: torch.Tensor, n_tokens: int, expert_ids: torch.Tensor, router_weights: torch.Tensor,
                      top_k: int, expert_table: redlite_moe_table, shared_expert: Optional[redlite_moe_expert],
                      out: torch.Tensor) -> int:
    return lib().redlite_moe_layer(_ptr(x), n_tokens, _ptr(expert_ids), _ptr(router_weights), top_k,
                                   ctypes.byref(expert_table),
                                   ctypes.byref(shared_expert) if shared_expert is not None else None, _ptr(out))


def redlite_moe_layer_noalloc(x: torch.Tensor, n_tokens: int, expert_ids: torch.Tensor, router_weights: torch.Tensor,
                              top_k: int, expert_table: redlite_moe_table, shared_expert: Optional[redlite_moe_expert],
                              out: torch.Tensor) -> int:
    """The layer without a caller workspace (scratch held by the library)."""
    return lib().redlite_moe_layer_noalloc(_ptr(x), n_tokens, _ptr(expert_ids), _ptr(router_weights), top_k,
                                           ctypes.byref(expert_table),
                                           ctypes.byref(shared_expert) if shared_expert is not None else None,
                                           _ptr(out))


def redlite_moe_layer_host(inputs_host: torch.Tensor, inputs_dev: torch.Tensor, n_tokens: int, top_k: int,
                           expert_table: redlite_moe_table, shared_expert: Optional[redlite_moe_expert],
                           out_dev: torch.Tensor, out_host: torch.Tensor) -> int:
    """The layer on inputs and output in host memory: one packed host -> device
    copy (x, ids, weights), the layer, the device -> host copy of out."""
    return lib().redlite_moe_layer_host(_ptr(inputs_host), _ptr(inputs_dev), n_tokens, top_k,
                                        ctypes.byref(expert_table),
                                        ctypes.byref(shared_expert) if shared_expert is not None else None,
                                        _ptr(out_dev), _ptr(out_host))


def redlite_moe_host_input_bytes(hidden: int, n_tokens: int, top_k: int) -> int:
    return int(lib().redlite_moe_host_input_bytes(hidden, n_tokens, top_k))


def redlite_moe_route_topk(logits: torch.Tensor, n_tokens: int, n_experts: int, top_k: int, expert_ids: torch.Tensor,
                           router_weights: torch.Tensor, stream=None) -> int:
    """The router: softmax over the logits, top-k by probability, renormalised weights."""
    return lib().redlite_moe_route_topk(_ptr(logits), n_tokens, n_experts, top_k, _ptr(expert_ids),
                                        _ptr(router_weights), _stream_handle(stream))


def redlite_moe_block_scratch_bytes(hidden: int, n_experts: int, max_tokens: int, top_k: int) -> int:
    return int(lib().redlite_moe_block_scratch_bytes(hidden, n_experts, max_tokens, top_k))


def redlite_moe_block(h: torch.Tensor, n_tokens: int, norm_weight: torch.Tensor, eps: float, router_w: torch.Tensor,
                      top_k: int, expert_table: redlite_moe_table, shared_expert: Optional[redlite_moe_expert],
                      out: torch.Tensor, scratch: torch.Tensor) -> int:
    """out = h + layer(RMSNorm(h)) with the router's own top-k routing."""
    return lib().redlite_moe_block(_ptr(h), n_tokens, _ptr(norm_weight), float(eps), _ptr(router_w), top_k,
                                   ctypes.byref(expert_table),
                                   ctypes.byref(shared_expert) if shared_expert is not None else None, _ptr(out),
                                   _ptr(scratch), scratch.numel() * scratch.element_size())


def redlite_moe_upload_experts(hidden: int, ids, host_experts, pool: torch.Tensor, pool_offset: int,
                               table_dev: torch.Tensor, n_experts: int, counters=None, stream=None):
    """ids: list of expert ids; host_experts: objects with qtype, ffn and numpy gate/up/down arrays.
    Returns (rc, pool_end)."""
    import numpy as np

    n = len(ids)
    ids_a = (ctypes.c_int32 * max(n, 1))(*[int(i) for i in ids])
    hx = (redlite_moe_expert * max(n, 1))()
    keep = []
    for i, ex in enumerate(host_experts):
        mats = [np.ascontiguousarray(m, dtype=np.uint8) for m in (ex.gate, ex.up, ex.down)]
        keep.extend(mats)
        hx[i] = redlite_moe_expert(int(ex.qtype), int(ex.ffn), *[m.ctypes.data for m in mats])
    end = ctypes.c_size_t(0)
    ctr = counters if counters is not None else redlite_moe_upload_counters()
    rc = lib().redlite_moe_upload_experts(hidden, ids_a, hx, n, _ptr(pool), pool.numel() * pool.element_size(),
                                          pool_offset, _ptr(table_dev), n_experts, _stream_handle(stream),
                                          ctypes.byref(ctr), ctypes.byref(end))
    del keep
    return rc, int(end.value)


def redlite_proj_matrix_bytes(qtype: int, rows: int, k: int) -> int:
    return int(lib().redlite_proj_matrix_bytes(qtype, rows, k))


def redlite_proj_gemv(qtype: int, W: torch.Tensor, rows: int, k: int, x: torch.Tensor, n_tokens: int,
                      y: torch.Tensor, stream=None) -> int:
    """y = W x for a Q8_0-style (3) or Q4_K-style (4) projection matrix."""
    return lib().redlite_proj_gemv(qtype, _ptr(W), rows, k, _ptr(x), n_tokens, _ptr(y), _stream_handle(stream))


class SlotPool:
    """The bounded, top-k-aware LRU slot pool (a host object of the library).
    plan() is the policy step alone (no device work); acquire() also copies
    the misses' matrices into their device slots and updates the slot table."""

    def __init__(self, n_experts: int, capacity: int):
        self.n_experts, self.capacity = n_experts, capacity
        self.handle = lib().redlite_moe_pool_create(n_experts, capacity)
        if not self.handle:
            raise RuntimeError("redlite_moe_pool_create failed")
        self.counters = redlite_moe_pool_counters()

    def close(self):
        if self.handle:
            lib().redlite_moe_pool_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def plan(self, ids):
        """(rc, slots, evicted, miss, token) for the selection `ids`."""
        import numpy as np

        a = np.ascontiguousarray(ids, dtype=np.int32)
        n = a.size
        slots = np.zeros(max(n, 1), np.int32)
        ev = np.zeros(max(n, 1), np.int32)
        miss = np.zeros(max(n, 1), np.uint8)
        tok = ctypes.c_int64(0)
        rc = lib().redlite_moe_pool_plan(self.handle, a.ctypes.data_as(_c_void_p), n, slots.ctypes.data_as(_c_void_p),
                                         ev.ctypes.data_as(_c_void_p), miss.ctypes.data_as(_c_void_p),
                                         ctypes.byref(tok))
        return rc, slots[:n].tolist(), ev[:n].tolist(), miss[:n].astype(bool).tolist(), tok.value

    def complete(self, token: int) -> int:
        return lib().redlite_moe_pool_complete(self.handle, token)

    def release(self, token: int, stream=None) -> int:
        return lib().redlite_moe_pool_release(self.handle, token, _stream_handle(stream))

    def slot_of(self, expert: int) -> int:
        return int(lib().redlite_moe_pool_slot_of(self.handle, expert))

    def pins(self, slot: int) -> int:
        return int(lib().redlite_moe_pool_pins(self.handle, slot))

    def acquire(self, ids, host_experts, hidden: int, slots: torch.Tensor, slot_bytes: int, table_dev: torch.Tensor,
                copy_stream, compute_stream):
        """host_experts: ctypes array [n_experts] of redlite_moe_expert with host pointers (resident layout).
        Returns (rc, token)."""
        import numpy as np

        a = np.ascontiguousarray(ids, dtype=np.int32)
        tok = ctypes.c_int64(0)
        rc = lib().redlite_moe_pool_acquire(self.handle, a.ctypes.data_as(_c_void_p), a.size,
                                            ctypes.cast(host_experts, _c_void_p), hidden, _ptr(slots), slot_bytes,
                                            _ptr(table_dev), _stream_handle(copy_stream),
                                            _stream_handle(compute_stream), ctypes.byref(self.counters),
                                            ctypes.byref(tok))
        return rc, tok.value


def launches_per_call(n_tokens: int, top_k: int, has_shared: bool, fast: bool = True) -> int:
    """Kernels one redlite_moe_layer call enqueues: the fused decode kernel for
    decode-sized calls on tiled tables; otherwise bucketing (count, plan,
    scatter), then on tiled tables the bf16 conversion of x and the gate/up and
    down tensor-core kernels, else the gate/up and down CUDA-core tiles."""
    if n_tokens == 0:
        return 0
    if fast and n_tokens * top_k <= 640 and (not has_shared or n_tokens <= 64):
        return 1
    return 6 if fast else 5
