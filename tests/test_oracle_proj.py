"""Pins of the oracle's projection formats (Q8_0-style, Q4_K-style): hand-
worked blocks (tests/golden/proj_examples.json), field locality (one field
changes exactly the weights it covers, by the amount the format states),
and the closed form of a constant matrix."""
import json
import os

import numpy as np
import pytest

import fixtures

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "proj_examples.json")


def test_golden_blocks(oracle_lib):
    for ex in json.load(open(GOLDEN))["examples"]:
        w = oracle_lib.dequant_proj(ex["qtype"], np.array(ex["bytes"], np.uint8), ex["rows"], ex["k"]).reshape(-1)
        for i, v in ex["weights"].items():
            assert w[int(i)] == v, (ex["why"], i, w[int(i)], v)


def test_q8_0_field_locality(oracle_lib):
    m = fixtures.make_proj_matrix(5, 3, 4, 256)
    base = oracle_lib.dequant_proj(3, m, 4, 256).reshape(-1)
    d = float(np.array([int(m[34 * 9]) | (int(m[34 * 9 + 1]) << 8)], np.uint16).view(np.float16)[0])
    m2 = m.copy()
    m2[34 * 9 + 2 + 7] = (int(m2[34 * 9 + 2 + 7]) + 1) & 0xFF  # q[7] of block 9, one step up (mod 256)
    w2 = oracle_lib.dequant_proj(3, m2, 4, 256).reshape(-1)
    diff = np.nonzero(w2 != base)[0]
    assert diff.tolist() == [9 * 32 + 7]
    old = int(np.int8(m[34 * 9 + 2 + 7]))
    new = int(np.int8(m2[34 * 9 + 2 + 7]))
    assert w2[9 * 32 + 7] - base[9 * 32 + 7] == d * (new - old)


def test_q4_k_field_locality(oracle_lib):
    m = fixtures.make_proj_matrix(6, 4, 2, 512)
    base = oracle_lib.dequant_proj(4, m, 2, 512).reshape(-1)
    blk = 3 * 144  # block 3 covers weights 768..1023
    # one nibble: weight 768 + 77 moves by d * scale(sub-block 2) * dq
    m2 = m.copy()
    m2[blk + 16 + 77 // 2] ^= 0x10  # toggles bit 0 of the high nibble (weight 77 is odd)
    w2 = oracle_lib.dequant_proj(4, m2, 2, 512).reshape(-1)
    assert np.nonzero(w2 != base)[0].tolist() == [768 + 77]
    # one minimum field: all 32 weights of sub-block 5 move by -dmin * dm, nothing else
    field = int.from_bytes(bytes(m[blk + 4:blk + 16]), "little")
    mn = (field >> (48 + 30)) & 63
    f2 = field ^ (1 << (48 + 30))
    m3 = m.copy()
    m3[blk + 4:blk + 16] = np.frombuffer(f2.to_bytes(12, "little"), np.uint8)
    w3 = oracle_lib.dequant_proj(4, m3, 2, 512).reshape(-1)
    changed = np.nonzero(w3 != base)[0]
    assert changed.tolist() == list(range(768 + 160, 768 + 192))
    dmin = float(np.array([int(m[blk + 2]) | (int(m[blk + 3]) << 8)], np.uint16).view(np.float16)[0])
    dm = ((f2 >> (48 + 30)) & 63) - mn
    np.testing.assert_allclose(w3[changed] - base[changed], -dmin * dm, rtol=0, atol=1e-12)


@pytest.mark.parametrize("qtype", [3, 4])
def test_constant_matrix_closed_form(oracle_lib, qtype):
    """Every block equal and encoding one constant c: y = c * sum(x) per row."""
    if qtype == 3:
        blk = np.array([0x00, 0x34] + [3] * 32, np.uint8)  # d = 0.25, q = 3: c = 0.75
        c, bw = 0.75, 32
    else:
        field = sum((5 << (6 * j)) | (1 << (48 + 6 * j)) for j in range(8))
        blk = np.array([0x00, 0x3C, 0x00, 0x38] + list(field.to_bytes(12, "little")) + [0x22] * 128, np.uint8)
        c, bw = 1.0 * 5 * 2 - 0.5 * 1, 256  # d=1, scale 5, q 2, dmin 0.5, min 1
    rows, k = 8, 512
    m = np.tile(blk, rows * k // bw)
    x = fixtures.make_x(12, 3, k)
    y = oracle_lib.gemv_proj(qtype, m, rows, k, x)
    want = c * x.astype(np.float64).sum(axis=1)
    np.testing.assert_allclose(y, np.repeat(want[:, None], rows, axis=1), rtol=1e-12)
