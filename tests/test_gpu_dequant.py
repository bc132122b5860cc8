"""Dequantised weights from the CUDA decoder are bit-exact against the oracle,
in fp32 and in bf16 (round to nearest even, applied by the oracle to its own
exact values)."""
import numpy as np
import pytest
import torch

import fixtures

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    from routed_expert_ffn_iq2_b200 import build

    build.build()
    import routed_expert_ffn_iq2_b200 as P

    return P


@pytest.fixture(scope="module")
def grids(P):
    w = fixtures.workload(2)
    g = torch.zeros(P.redlite_moe_grids_bytes(), dtype=torch.uint8, device="cuda")
    assert P.redlite_moe_expand_grids(w.grid_iq2, w.grid_iq1, g) == 0
    return w, g


def _gpu_dequant(P, g, qtype, packed, rows, k):
    dev = torch.from_numpy(P.redlite_moe_pack_matrix(qtype, rows, k, packed)).cuda()
    f = torch.empty(rows * k, dtype=torch.float32, device="cuda")
    b = torch.empty(rows * k, dtype=torch.int16, device="cuda")
    assert P.redlite_moe_dequant(qtype, dev, rows, k, g, f, b) == 0
    torch.cuda.synchronize()
    return f.cpu().numpy(), b.cpu().numpy().view(np.uint16)


def _edge_blocks(qtype, n):
    """Extremes: smallest/largest normal fp16 d, every sub-scale 0 or max, all signs/deltas set or clear."""
    bb = fixtures.BLOCK_BYTES[qtype]
    st = fixtures.Stream(99, qtype)
    out = st.bytes(n * bb).reshape(n, bb)
    for i in range(n):
        d = [0x0400, 0x7BFF, 0x3C00, 0x0001][i % 4]
        out[i, 0], out[i, 1] = d & 0xFF, d >> 8
        if qtype == 1:
            out[i, 2:6] = 0x00 if i % 2 else 0xFF
            out[i, 42:74] = 0xFF if i % 3 == 0 else out[i, 42:74]
        else:
            out[i, 50:56] = 0x00 if i % 2 else 0xFF
            out[i, 34:50] = 0x88 if i % 3 == 0 else out[i, 34:50]
    return out.reshape(-1)


@pytest.mark.parametrize("qtype,rows,k", [(1, 64, 2048), (2, 64, 2048), (1, 256, 64), (2, 2048, 512), (1, 3, 256),
                                          (2, 128, 128), (1, 48, 768), (2, 32, 256)])
def test_dequant_bit_exact(P, grids, oracle_lib, qtype, rows, k):
    w, g = grids
    packed = fixtures.make_matrix(17, qtype, rows, k, 5)
    grid = oracle_lib.expand_grid(qtype, w.grid_iq2 if qtype == 1 else w.grid_iq1)
    ref = oracle_lib.dequant_matrix(qtype, packed, rows, k, grid).reshape(-1)
    f, b = _gpu_dequant(P, g, qtype, packed, rows, k)
    np.testing.assert_array_equal(f.astype(np.float64), ref)
    np.testing.assert_array_equal(b, oracle_lib.float_to_bf16(ref.astype(np.float32)))


@pytest.mark.parametrize("qtype", [1, 2])
def test_dequant_edge_blocks_bit_exact(P, grids, oracle_lib, qtype):
    w, g = grids
    packed = _edge_blocks(qtype, 16)
    grid = oracle_lib.expand_grid(qtype, w.grid_iq2 if qtype == 1 else w.grid_iq1)
    ref = oracle_lib.dequant_matrix(qtype, packed, 16, 256, grid).reshape(-1)
    f, b = _gpu_dequant(P, g, qtype, packed, 16, 256)
    np.testing.assert_array_equal(f.astype(np.float64), ref)
    np.testing.assert_array_equal(b, oracle_lib.float_to_bf16(ref.astype(np.float32)))


def test_grid_expansion_on_device(P, grids, oracle_lib):
    """The device grid buffer's int8 values equal the oracle's expansion."""
    w, g = grids
    host = g.cpu().numpy()
    np.testing.assert_array_equal(host[:4096].view(np.int8), oracle_lib.expand_grid(1, w.grid_iq2))
    np.testing.assert_array_equal(host[4096:4096 + 16384].view(np.int8), oracle_lib.expand_grid(2, w.grid_iq1))
