"""Host-side conversion to the resident tiled layout (pure host code, no GPU):
the documented field positions of include/redlite_moe.h's resident layout are
checked against the interchange bytes they came from."""
import numpy as np
import pytest

import fixtures


@pytest.fixture(scope="module")
def P():
    from routed_expert_ffn_iq2_b200 import build

    build.build()
    import routed_expert_ffn_iq2_b200 as P

    return P


def test_untiled_shapes_unchanged(P):
    m = fixtures.make_matrix(1, 1, 256, 64, 0)
    np.testing.assert_array_equal(P.redlite_moe_pack_matrix(1, 256, 64, m), m)
    m = fixtures.make_matrix(1, 2, 8, 256, 0)  # 8 rows: not a whole 16-row tile
    np.testing.assert_array_equal(P.redlite_moe_pack_matrix(2, 8, 256, m), m)


@pytest.mark.parametrize("rows,k", [(32, 512), (16, 256)])
def test_iq2_tile_fields(P, rows, k):
    m = fixtures.make_matrix(2, 1, rows, k, 0)
    t = P.redlite_moe_pack_matrix(1, rows, k, m)
    assert t.size == m.size and not np.array_equal(t, m)
    nkb = k // 256
    for r in range(rows):
        for kb in range(nkb):
            blk = m[(r * nkb + kb) * 74:(r * nkb + kb + 1) * 74]
            tb = t[((r // 16) * nkb + kb) * 1184:((r // 16) * nkb + kb + 1) * 1184]
            rr = r % 16
            q, h = rr % 8, rr // 8
            for g in range(32):
                L, i = 4 * q + (g & 3), 2 * (g >> 2) + h
                assert tb[32 * L + i] == blk[6 + g]
                sw = int.from_bytes(bytes(tb[32 * L + 16 + 4 * (i // 4):32 * L + 20 + 4 * (i // 4)]), "little")
                assert sum(((sw >> (4 * j + i % 4)) & 1) << j for j in range(8)) == blk[42 + g]
                qh = int(tb[1024 + 2 * L]) | (int(tb[1025 + 2 * L]) << 8)
                assert (qh >> i) & 1 == (blk[38 + g // 8] >> (g % 8)) & 1
            assert bytes(tb[1088 + 8 * q + 4 * h:1088 + 8 * q + 4 * h + 4]) == bytes(blk[2:6])
            assert bytes(tb[1152 + 4 * q + 2 * h:1152 + 4 * q + 2 * h + 2]) == bytes(blk[0:2])


def test_iq1_tile_fields(P):
    rows, k = 16, 512
    m = fixtures.make_matrix(3, 2, rows, k, 0)
    t = P.redlite_moe_pack_matrix(2, rows, k, m)
    nkb = 2
    for r in range(rows):
        for kb in range(nkb):
            blk = m[(r * nkb + kb) * 56:(r * nkb + kb + 1) * 56]
            tb = t[kb * 896:(kb + 1) * 896]
            q, h = r % 8, r // 8
            for g in range(32):
                base, i = 48 * (2 * q + (g & 1)), 2 * (g >> 1) + h
                assert tb[base + i] == blk[2 + g]
                nib = (tb[base + 32 + i // 2] >> (4 * (i & 1))) & 15
                assert nib == (blk[34 + g // 2] >> (4 * (g % 2))) & 15
            assert bytes(tb[768 + 12 * q + 6 * h:768 + 12 * q + 6 * h + 6]) == bytes(blk[50:56])
            assert bytes(tb[864 + 4 * q + 2 * h:864 + 4 * q + 2 * h + 2]) == bytes(blk[0:2])


def test_pack_rejects(P):
    import ctypes

    L = P.lib()
    buf = np.zeros(1024, np.uint8)
    p = buf.ctypes.data_as(ctypes.c_void_p)
    assert L.redlite_moe_pack_matrix(3, 16, 256, p, buf[512:].ctypes.data_as(ctypes.c_void_p)) == P.REDLITE_EINVAL
    assert L.redlite_moe_pack_matrix(1, 16, 300, p, buf[512:].ctypes.data_as(ctypes.c_void_p)) == P.REDLITE_EUNSUPPORTED
    assert L.redlite_moe_pack_matrix(1, 16, 256, p, p) == P.REDLITE_EINVAL
