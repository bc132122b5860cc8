"""ctypes front end of the CPU oracle (plain C, fp64).

TEST INFRASTRUCTURE ONLY: imported by the test suite, the smoke check and the
benchmark's CPU-baseline leg.  The CUDA library and its Python binding never
import this package.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "redlite_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

QTYPE_IQ2XS = 1
QTYPE_IQ1M = 2
QTYPE_Q8_0 = 3
QTYPE_Q4_K = 4
OK = 0
EINVAL = -1
SKIPPED_PAIRS = 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP).  Returns the library path."""
    hdr = os.path.join(_HERE, "redlite_oracle.h")
    if not force and os.path.exists(_LIB):
        newest = max(os.path.getmtime(_SRC), os.path.getmtime(hdr))
        if os.path.getmtime(_LIB) >= newest:
            return _LIB
    tmp = _LIB + ".tmp"
    subprocess.check_call(
        ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    )
    os.replace(tmp, _LIB)
    return _LIB


class _Expert(ctypes.Structure):
    _fields_ = [
        ("qtype", ctypes.c_int32),
        ("ffn", ctypes.c_int32),
        ("gate", ctypes.c_void_p),
        ("up", ctypes.c_void_p),
        ("down", ctypes.c_void_p),
    ]


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.oracle_block_bytes.argtypes = [ctypes.c_int]
        L.oracle_expand_grid.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
        L.oracle_fp16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_fp16_to_double.restype = ctypes.c_double
        L.oracle_float_to_bf16_rne.argtypes = [ctypes.c_float]
        L.oracle_float_to_bf16_rne.restype = ctypes.c_uint16
        L.oracle_shape_ok.argtypes = [ctypes.c_int64, ctypes.c_int64]
        L.oracle_dequant_matrix.argtypes = [
            ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
        ]
        L.oracle_moe_layer.argtypes = [
            ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
            ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ]
        L.oracle_set_threads.argtypes = [ctypes.c_int]
        L.oracle_dequant_proj.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                          ctypes.c_void_p]
        L.oracle_gemv_proj.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                       ctypes.c_int, ctypes.c_void_p]
        L.oracle_route_topk.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                        ctypes.c_void_p]
        L.oracle_moe_block.argtypes = [
            ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_double, ctypes.c_void_p,
            ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ]
        _lib = L
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def expand_grid(qtype: int, compact: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(compact, dtype=np.uint16)
    out = np.zeros(c.size * 8, dtype=np.int8)
    rc = lib().oracle_expand_grid(qtype, _ptr(c), c.size, _ptr(out))
    if rc != OK:
        raise ValueError(f"oracle_expand_grid failed ({rc})")
    return out


def expand_grid_rc(qtype: int, compact: np.ndarray) -> int:
    c = np.ascontiguousarray(compact, dtype=np.uint16)
    out = np.zeros(max(c.size, 1) * 8, dtype=np.int8)
    return lib().oracle_expand_grid(qtype, _ptr(c), c.size, _ptr(out))


def fp16_to_double(h: int) -> float:
    return lib().oracle_fp16_to_double(h)


def float_to_bf16(a: np.ndarray) -> np.ndarray:
    f = lib().oracle_float_to_bf16_rne
    flat = np.asarray(a, dtype=np.float32).reshape(-1)
    return np.array([f(float(v)) for v in flat], dtype=np.uint16).reshape(np.shape(a))


def shape_ok(rows: int, k: int) -> bool:
    return bool(lib().oracle_shape_ok(rows, k))


def dequant_matrix(qtype: int, packed: np.ndarray, rows: int, k: int, grid: np.ndarray) -> np.ndarray:
    p = np.ascontiguousarray(packed, dtype=np.uint8)
    g = np.ascontiguousarray(grid, dtype=np.int8)
    out = np.zeros(rows * k, dtype=np.float64)
    rc = lib().oracle_dequant_matrix(qtype, _ptr(p), rows, k, _ptr(g), _ptr(out))
    if rc != OK:
        raise ValueError(f"oracle_dequant_matrix failed ({rc})")
    return out.reshape(rows, k)


class ExpertSet:
    """Host descriptors for oracle_moe_layer; keeps the numpy buffers alive."""

    def __init__(self, experts: Sequence):
        self._keep = []
        self.arr = (_Expert * max(len(experts), 1))()
        for i, ex in enumerate(experts):
            if ex is None:
                self.arr[i] = _Expert(0, 0, None, None, None)
                continue
            bufs = [np.ascontiguousarray(m, dtype=np.uint8) for m in (ex.gate, ex.up, ex.down)]
            self._keep.extend(bufs)
            self.arr[i] = _Expert(ex.qtype, ex.ffn, *[b.ctypes.data for b in bufs])

    @property
    def ptr(self):
        return ctypes.cast(self.arr, ctypes.c_void_p)


def moe_layer(x, ids, weights, experts: Sequence, shared=None, grid_iq2=None, grid_iq1=None,
              hidden: Optional[int] = None, return_rc: bool = False):
    """Run the fp64 oracle layer.  `experts` is a list indexed by expert id (None = absent);
    grids are expanded int8 arrays.  Returns out [T, H] float64 (and the return code)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    T = x.shape[0]
    H = x.shape[1] if hidden is None else hidden
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    k = ids.shape[-1] if ids.ndim == 2 else (ids.size // max(T, 1))
    ids = ids.reshape(T, k)
    weights = np.ascontiguousarray(weights, dtype=np.float32).reshape(T, k)
    es = ExpertSet(experts)
    sh = ExpertSet([shared]) if shared is not None else None
    g2 = None if grid_iq2 is None else np.ascontiguousarray(grid_iq2, dtype=np.int8)
    g1 = None if grid_iq1 is None else np.ascontiguousarray(grid_iq1, dtype=np.int8)
    out = np.zeros((T, H), dtype=np.float64)
    rc = lib().oracle_moe_layer(
        _ptr(x), T, H, _ptr(ids), _ptr(weights), k, len(experts), es.ptr,
        sh.ptr if sh is not None else None, _ptr(g2), _ptr(g1), _ptr(out),
    )
    if rc < 0:
        raise ValueError(f"oracle_moe_layer failed ({rc})")
    return (out, rc) if return_rc else out


def set_threads(n: int) -> int:
    return lib().oracle_set_threads(n)


def workload_layer(w, tokens: Optional[Sequence[int]] = None):
    """Oracle output of a fixtures.Workload (optionally only for some token rows)."""
    experts = [None] * w.n_experts
    for e in w.selected():
        experts[e] = w.expert(e)
    x, ids, wt = w.x, w.ids, w.weights
    if tokens is not None:
        tokens = np.asarray(tokens)
        x, ids, wt = x[tokens], ids[tokens], wt[tokens]
    return moe_layer(x, ids, wt, experts, w.shared(), expand_grid(QTYPE_IQ2XS, w.grid_iq2),
                     expand_grid(QTYPE_IQ1M, w.grid_iq1))


def route_topk(logits, top_k: int):
    """The oracle router: (ids int32 [T, k], weights float64 [T, k]) from float logits [T, E]."""
    lg = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = lg.shape
    ids = np.zeros((T, top_k), dtype=np.int32)
    w = np.zeros((T, top_k), dtype=np.float64)
    rc = lib().oracle_route_topk(_ptr(lg), T, E, top_k, _ptr(ids), _ptr(w))
    if rc != OK:
        raise ValueError(f"oracle_route_topk failed ({rc})")
    return ids, w


def moe_block(h, gamma, eps: float, router_w, top_k: int, experts: Sequence, shared=None, grid_iq2=None,
              grid_iq1=None, return_routing: bool = False):
    """The oracle block out = h + layer(RMSNorm(h)) with its own routing; float64 [T, H]
    (and the routing ids / weights when asked)."""
    h = np.ascontiguousarray(h, dtype=np.float32)
    T, H = h.shape
    g = np.ascontiguousarray(gamma, dtype=np.float32)
    rw = np.ascontiguousarray(router_w, dtype=np.float32)
    E = rw.shape[0]
    es = ExpertSet(experts)
    sh = ExpertSet([shared]) if shared is not None else None
    g2 = None if grid_iq2 is None else np.ascontiguousarray(grid_iq2, dtype=np.int8)
    g1 = None if grid_iq1 is None else np.ascontiguousarray(grid_iq1, dtype=np.int8)
    out = np.zeros((T, H), dtype=np.float64)
    ids = np.zeros((T, top_k), dtype=np.int32)
    w = np.zeros((T, top_k), dtype=np.float64)
    rc = lib().oracle_moe_block(_ptr(h), T, H, _ptr(g), float(eps), _ptr(rw), E, top_k, es.ptr,
                                sh.ptr if sh is not None else None, _ptr(g2), _ptr(g1), _ptr(out), _ptr(ids), _ptr(w))
    if rc < 0:
        raise ValueError(f"oracle_moe_block failed ({rc})")
    return (out, ids, w) if return_routing else out


def dequant_proj(qtype: int, packed, rows: int, k: int) -> np.ndarray:
    """Weights of a Q8_0-style (3) or Q4_K-style (4) matrix as float64 [rows, k]."""
    p = np.ascontiguousarray(packed, dtype=np.uint8)
    out = np.zeros(rows * k, dtype=np.float64)
    rc = lib().oracle_dequant_proj(qtype, _ptr(p), rows, k, _ptr(out))
    if rc != OK:
        raise ValueError(f"oracle_dequant_proj failed ({rc})")
    return out.reshape(rows, k)


def gemv_proj(qtype: int, packed, rows: int, k: int, x) -> np.ndarray:
    """y = W x (float64 [n_tokens, rows]) for a projection-format matrix."""
    p = np.ascontiguousarray(packed, dtype=np.uint8)
    xv = np.ascontiguousarray(x, dtype=np.float32).reshape(-1, k)
    y = np.zeros((xv.shape[0], rows), dtype=np.float64)
    rc = lib().oracle_gemv_proj(qtype, _ptr(p), rows, k, _ptr(xv), xv.shape[0], _ptr(y))
    if rc != OK:
        raise ValueError(f"oracle_gemv_proj failed ({rc})")
    return y
