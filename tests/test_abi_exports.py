"""The C-ABI library loads without a GPU and exports every entry point that
include/redlite_moe.h declares; host-only argument checks answer without
touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names |= set(re.findall(r"^\s*(?:[\w\s\*]+?)\b(redlite_\w+)\s*\(", txt, flags=re.M))
    return names


@pytest.fixture(scope="module")
def native():
    from routed_expert_ffn_iq2_b200 import build

    build.build()
    import routed_expert_ffn_iq2_b200 as P

    return P


def test_every_declared_symbol_exported(native):
    declared = _declared()
    assert len(declared) >= 8
    lib = native.lib()
    for name in declared:
        assert hasattr(lib, name), name
    assert declared == set(native.EXPORTS), (declared ^ set(native.EXPORTS))


def test_host_only_sizes(native):
    assert native.redlite_moe_matrix_bytes(1, 512, 2048) == 303104
    assert native.redlite_moe_matrix_bytes(2, 512, 2048) == 229376
    assert native.redlite_moe_matrix_bytes(1, 2048, 512) == 303104
    assert native.redlite_moe_matrix_bytes(1, 256, 64) == 64 * 74
    assert native.redlite_moe_matrix_bytes(1, 256, 48) == 0
    assert native.redlite_moe_matrix_bytes(3, 512, 2048) == 0
    assert native.redlite_moe_grids_bytes() >= 512 * 8 + 2048 * 8
    assert native.redlite_moe_workspace_bytes(2048, 512, 64, 10, 512) > 64 * 11 * 512 * 4
    assert native.redlite_moe_workspace_bytes(0, 512, 64, 10, 512) == 0


def test_expand_grids_rejects_symbol3_before_device_work(native):
    g2 = np.zeros(512, np.uint16)
    g1 = np.zeros(2048, np.uint16)
    g2[7] = 0x0300
    rc = native.lib().redlite_moe_expand_grids(g2.ctypes.data_as(ctypes.c_void_p), g1.ctypes.data_as(ctypes.c_void_p),
                                               ctypes.c_void_p(256), None)
    assert rc == native.REDLITE_EINVAL
    rc = native.lib().redlite_moe_expand_grids(None, g1.ctypes.data_as(ctypes.c_void_p), ctypes.c_void_p(256), None)
    assert rc == native.REDLITE_EINVAL


def test_layer_rejects_bad_arguments_on_host(native):
    L = native.lib()
    t = native.redlite_moe_table(2048, 512, 512, 64, 0, 0, 0x1000, 0x2000, 0x3000, 1 << 30, 0x4000, None)
    p = ctypes.c_void_p(0x10000)
    # null table
    assert L.redlite_moe_layer(p, 1, p, p, 10, None, None, p) == native.REDLITE_EINVAL
    # top_k out of range
    assert L.redlite_moe_layer(p, 1, p, p, 0, ctypes.byref(t), None, p) == native.REDLITE_EINVAL
    assert L.redlite_moe_layer(p, 1, p, p, 17, ctypes.byref(t), None, p) == native.REDLITE_EINVAL
    # n_tokens above the table's limit, negative
    assert L.redlite_moe_layer(p, 65, p, p, 10, ctypes.byref(t), None, p) == native.REDLITE_EINVAL
    assert L.redlite_moe_layer(p, -1, p, p, 10, ctypes.byref(t), None, p) == native.REDLITE_EINVAL
    # zero tokens: nothing to do
    assert L.redlite_moe_layer(None, 0, None, None, 10, ctypes.byref(t), None, None) == native.REDLITE_OK
    # null tensors
    assert L.redlite_moe_layer(None, 1, p, p, 10, ctypes.byref(t), None, p) == native.REDLITE_EINVAL
    # misaligned x
    assert L.redlite_moe_layer(ctypes.c_void_p(0x10004), 1, p, p, 10, ctypes.byref(t), None, p) == native.REDLITE_EINVAL
    # workspace too small
    t2 = native.redlite_moe_table(2048, 512, 512, 64, 0, 0, 0x1000, 0x2000, 0x3000, 1024, 0x4000, None)
    assert L.redlite_moe_layer(p, 1, p, p, 10, ctypes.byref(t2), None, p) == native.REDLITE_ENOMEM
    # bad shared expert (bad qtype / unsupported shape)
    sh = native.redlite_moe_expert(3, 512, 0x1000, 0x2000, 0x3000)
    assert L.redlite_moe_layer(p, 1, p, p, 10, ctypes.byref(t), ctypes.byref(sh), p) == native.REDLITE_EINVAL
    sh = native.redlite_moe_expert(1, 48, 0x1000, 0x2000, 0x3000)
    assert L.redlite_moe_layer(p, 1, p, p, 10, ctypes.byref(t), ctypes.byref(sh), p) == native.REDLITE_EINVAL
    # hidden not a multiple of 32
    t3 = native.redlite_moe_table(2047, 512, 512, 64, 0, 0, 0x1000, 0x2000, 0x3000, 1 << 30, 0x4000, None)
    assert L.redlite_moe_layer(p, 1, p, p, 10, ctypes.byref(t3), None, p) == native.REDLITE_EINVAL


def test_dequant_rejects_on_host(native):
    L = native.lib()
    p = ctypes.c_void_p(0x10000)
    assert L.redlite_moe_dequant(3, p, 1, 256, p, p, None, None) == native.REDLITE_EINVAL
    assert L.redlite_moe_dequant(1, p, 1, 300, p, p, None, None) == native.REDLITE_EUNSUPPORTED
    assert L.redlite_moe_dequant(1, p, 1, 256, p, None, None, None) == native.REDLITE_EINVAL


def _shared_cases(native):
    """Shared-expert descriptors no layer kernel may be handed, each with why."""
    E = native.redlite_moe_expert
    return [
        (E(3, 512, 0x1000, 0x2000, 0x3000), "unknown qtype"),
        (E(1, 0, 0x1000, 0x2000, 0x3000), "zero width"),
        (E(1, -256, 0x1000, 0x2000, 0x3000), "negative width"),
        (E(1, 1024, 0x1000, 0x2000, 0x3000), "wider than max_ffn"),
        (E(1, 512, 0x1004, 0x2000, 0x3000), "gate not 16-byte aligned"),
        (E(2, 512, 0x1000, 0x2008, 0x3000), "up not 16-byte aligned"),
        (E(1, 512, 0x1000, 0x2000, 0x3001), "down not 16-byte aligned"),
        (E(1, 512, 0x1000, None, 0x3000), "null up"),
        (E(1, 48, 0x1000, 0x2000, 0x3000), "width the packed layout does not take"),
    ]


def test_layer_rejects_bad_shared_expert_on_both_paths(native):
    """Every malformed shared expert returns EINVAL before any device work,
    whichever path the table selects; on the tiled path (min_ffn >= 256) a
    width that is not a multiple of 256, or below the declared min_ffn, is
    malformed too."""
    L = native.lib()
    p = ctypes.c_void_p(0x10000)
    for min_ffn in (0, 256):
        t = native.redlite_moe_table(2048, 512, 512, 64, min_ffn, 0, 0x1000, 0x2000, 0x3000, 1 << 30, 0x4000, None)
        for sh, why in _shared_cases(native):
            rc = L.redlite_moe_layer(p, 1, p, p, 10, ctypes.byref(t), ctypes.byref(sh), p)
            assert rc == native.REDLITE_EINVAL, (min_ffn, why, rc)
    t = native.redlite_moe_table(2048, 512, 512, 64, 512, 0, 0x1000, 0x2000, 0x3000, 1 << 30, 0x4000, None)
    for sh in (native.redlite_moe_expert(1, 128, 0x1000, 0x2000, 0x3000),   # valid shape, not tiled
               native.redlite_moe_expert(1, 256, 0x1000, 0x2000, 0x3000)):  # below the declared min_ffn
        assert L.redlite_moe_layer(p, 1, p, p, 10, ctypes.byref(t), ctypes.byref(sh), p) == native.REDLITE_EINVAL


def test_no_alloc_rejects_on_host(native):
    """The allocation-free entry point validates the shared expert like the
    fused path of redlite_moe_layer, and refuses a call whose scratch does not
    fit its fixed array with ENOMEM before it touches the device (without a
    GPU any device call would return ECUDA instead)."""
    L = native.lib()
    p = ctypes.c_void_p(0x10000)
    t = native.redlite_moe_table(2048, 512, 512, 64, 512, 0, 0x1000, 0x2000, 0x3000, 0, 0x4000, None)
    for sh, why in _shared_cases(native) + [(native.redlite_moe_expert(1, 128, 0x1000, 0x2000, 0x3000), "not tiled")]:
        rc = L.redlite_moe_layer_noalloc(p, 1, p, p, 10, ctypes.byref(t), ctypes.byref(sh), p)
        assert rc == native.REDLITE_EINVAL, (why, rc)
    # 64 tokens x top-10 + shared at width 2048: 704 pairs x 2048 fp32 h values > 4 MiB
    big = native.redlite_moe_table(2048, 512, 2048, 64, 2048, 0, 0x1000, 0x2000, 0x3000, 0, 0x4000, None)
    sh = native.redlite_moe_expert(1, 2048, 0x1000, 0x2000, 0x3000)
    assert L.redlite_moe_layer_noalloc(p, 64, p, p, 10, ctypes.byref(big), ctypes.byref(sh), p) == native.REDLITE_ENOMEM
    # widths the fused kernel does not take
    t1 = native.redlite_moe_table(256, 16, 64, 1, 64, 0, 0x1000, 0x2000, 0x3000, 0, 0x4000, None)
    assert L.redlite_moe_layer_noalloc(p, 1, p, p, 4, ctypes.byref(t1), None, p) == native.REDLITE_EUNSUPPORTED


def test_host_buffer_layer_rejects_on_host(native):
    """The host-buffer entry point refuses null or misaligned buffers, a bad
    shared expert and an undersized workspace before it enqueues anything
    (without a GPU any copy or launch would return ECUDA instead), and a
    zero-token call is a no-op."""
    L = native.lib()
    h = ctypes.c_void_p(0x20000)
    d = ctypes.c_void_p(0x10000)
    t = native.redlite_moe_table(2048, 512, 512, 64, 512, 0, 0x1000, 0x2000, 0x3000, 1 << 30, 0x4000, None)
    T = ctypes.byref(t)
    assert L.redlite_moe_layer_host(h, d, 0, 10, T, None, d, h) == native.REDLITE_OK
    assert L.redlite_moe_layer_host(None, d, 1, 10, T, None, d, h) == native.REDLITE_EINVAL
    assert L.redlite_moe_layer_host(h, None, 1, 10, T, None, d, h) == native.REDLITE_EINVAL
    assert L.redlite_moe_layer_host(h, d, 1, 10, T, None, None, h) == native.REDLITE_EINVAL
    assert L.redlite_moe_layer_host(h, d, 1, 10, T, None, d, None) == native.REDLITE_EINVAL
    assert L.redlite_moe_layer_host(h, ctypes.c_void_p(0x10008), 1, 10, T, None, d, h) == native.REDLITE_EINVAL
    assert L.redlite_moe_layer_host(h, d, 1, 10, T, None, ctypes.c_void_p(0x10004), h) == native.REDLITE_EINVAL
    assert L.redlite_moe_layer_host(h, d, 65, 10, T, None, d, h) == native.REDLITE_EINVAL  # > max_tokens
    assert L.redlite_moe_layer_host(h, d, 1, 17, T, None, d, h) == native.REDLITE_EINVAL  # top_k
    for sh, why in _shared_cases(native):
        assert L.redlite_moe_layer_host(h, d, 1, 10, T, ctypes.byref(sh), d, h) == native.REDLITE_EINVAL, why
    small = native.redlite_moe_table(2048, 512, 512, 64, 512, 0, 0x1000, 0x2000, 0x3000, 4096, 0x4000, None)
    assert L.redlite_moe_layer_host(h, d, 1, 10, ctypes.byref(small), None, d, h) == native.REDLITE_ENOMEM
    # the packed input buffer: x, then ids, then weights
    assert L.redlite_moe_host_input_bytes(2048, 64, 10) == 4 * (2048 + 20) * 64
    assert L.redlite_moe_host_input_bytes(2048, 0, 10) == 0


def test_router_and_block_reject_on_host(native):
    L = native.lib()
    p = ctypes.c_void_p(0x10000)
    for T, E, k in [(1, 16, 17), (1, 16, 0), (1, 8, 9), (1, 1025, 4), (1, 0, 1), (-1, 16, 4)]:
        assert L.redlite_moe_route_topk(p, T, E, k, p, p, None) == native.REDLITE_EINVAL, (T, E, k)
    assert L.redlite_moe_route_topk(p, 0, 512, 10, None, None, None) == native.REDLITE_OK
    assert L.redlite_moe_route_topk(None, 1, 512, 10, p, p, None) == native.REDLITE_EINVAL
    t = native.redlite_moe_table(2048, 512, 512, 64, 512, 0, 0x1000, 0x2000, 0x3000, 1 << 30, 0x4000, None)
    need = native.redlite_moe_block_scratch_bytes(2048, 512, 64, 10)
    assert need >= 64 * 2048 * 4 + 64 * 512 * 4
    assert L.redlite_moe_block(p, 4, p, ctypes.c_float(1e-6), p, 10, ctypes.byref(t), None, p, p, need - 1) == \
        native.REDLITE_ENOMEM
    assert L.redlite_moe_block(p, 4, p, ctypes.c_float(1e-6), p, 10, ctypes.byref(t), None,
                               ctypes.c_void_p(0x10004), p, need) == native.REDLITE_EINVAL
    assert L.redlite_moe_block(p, 65, p, ctypes.c_float(1e-6), p, 10, ctypes.byref(t), None, p, p, need) == \
        native.REDLITE_EINVAL
    assert L.redlite_moe_block(p, 4, p, ctypes.c_float(-1.0), p, 10, ctypes.byref(t), None, p, p, need) == \
        native.REDLITE_EINVAL
    assert L.redlite_moe_block(None, 0, None, ctypes.c_float(1e-6), None, 10, ctypes.byref(t), None, None, None, 0) == \
        native.REDLITE_OK


def test_proj_gemv_rejects_on_host(native):
    L = native.lib()
    p = ctypes.c_void_p(0x10000)
    assert native.redlite_proj_matrix_bytes(3, 64, 2048) == 64 * 64 * 34
    assert native.redlite_proj_matrix_bytes(4, 2048, 4096) == 2048 * 16 * 144
    assert native.redlite_proj_matrix_bytes(4, 8, 300) == 0 and native.redlite_proj_matrix_bytes(1, 8, 256) == 0
    assert L.redlite_proj_gemv(4, p, 8, 300, p, 1, p, None) == native.REDLITE_EUNSUPPORTED
    assert L.redlite_proj_gemv(4, p, 8, 256, p, 9, p, None) == native.REDLITE_EINVAL
    assert L.redlite_proj_gemv(5, p, 8, 256, p, 1, p, None) == native.REDLITE_EINVAL
    assert L.redlite_proj_gemv(4, ctypes.c_void_p(0x10008), 8, 256, p, 1, p, None) == native.REDLITE_EINVAL
    assert L.redlite_proj_gemv(3, ctypes.c_void_p(0x10001), 8, 256, p, 1, p, None) == native.REDLITE_EINVAL
    assert L.redlite_proj_gemv(4, p, 8, 256, p, 0, p, None) == native.REDLITE_OK
