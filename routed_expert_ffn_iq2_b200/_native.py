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
REDLITE_OK = 0
REDLITE_EINVAL = -1
REDLITE_EUNSUPPORTED = -2
REDLITE_ENOMEM = -3
REDLITE_ECUDA = -4
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
