"""Pins of the oracle's block dequantisation.

(1) hand-assembled blocks with hand-worked weights (tests/golden/dequant_examples.json);
(2) locality properties on random blocks: changing one field changes exactly the
weights that field governs, by exactly the factor the format implies.  A wrong
offset, index or sub-block mapping moves the change elsewhere and fails."""
import json
import os

import numpy as np
import pytest

import fixtures

GOLD = os.path.join(os.path.dirname(__file__), "golden", "dequant_examples.json")


def _grid_from(spec, qtype, oracle_lib):
    n = {1: 512, 2: 2048}[qtype]
    compact = np.full(n, int(spec["grid_default"], 16), np.uint16)
    for k, v in spec["grid"].items():
        compact[int(k)] = int(v, 16)
    return oracle_lib.expand_grid(qtype, compact)


def _bytes_from(spec):
    b = np.zeros(spec["nbytes"], np.uint8)
    for k, v in spec["bytes"].items():
        b[int(k)] = int(v, 16)
    return b


@pytest.mark.parametrize("idx", range(4))
def test_dequant_golden(oracle_lib, idx):
    spec = json.load(open(GOLD))["blocks"][idx]
    q = spec["qtype"]
    w = oracle_lib.dequant_matrix(q, _bytes_from(spec), 1, 256, _grid_from(spec, q, oracle_lib))[0]
    for pos, val in spec["expect"].items():
        assert w[int(pos)] == val, (spec["name"], pos, w[int(pos)], val)
    size = spec["default_by_subblock"]["size"]
    vals = spec["default_by_subblock"]["values"]
    special = set(spec["special_groups"])
    for j in range(256):
        if j // 8 in special:
            continue
        assert w[j] == vals[j // size], (spec["name"], j, w[j], vals[j // size])


def _rand_block(qtype, seed):
    return fixtures.make_matrix(seed, qtype, 1, 256, 77).copy()


def _grids():
    w = fixtures.workload(2)
    return w.grid_iq2, w.grid_iq1


def _deq(oracle_lib, qtype, blk):
    g2, g1 = _grids()
    grid = oracle_lib.expand_grid(qtype, g2 if qtype == 1 else g1)
    return oracle_lib.dequant_matrix(qtype, blk, 1, 256, grid)[0]


@pytest.mark.parametrize("seed", range(6))
def test_iq2_sign_bit_negates_one_weight(oracle_lib, seed):
    blk = _rand_block(1, seed)
    base = _deq(oracle_lib, 1, blk)
    for g, j in [(0, 0), (3, 7), (17, 2), (31, 5)]:
        b2 = blk.copy()
        b2[42 + g] ^= 1 << j
        w2 = _deq(oracle_lib, 1, b2)
        diff = np.nonzero(w2 != base)[0]
        assert diff.tolist() == [8 * g + j]
        assert w2[8 * g + j] == -base[8 * g + j]


@pytest.mark.parametrize("seed", range(6))
def test_iq2_subscale_governs_32_weights(oracle_lib, seed):
    blk = _rand_block(1, seed)
    base = _deq(oracle_lib, 1, blk)
    for sub in range(8):
        b2 = blk.copy()
        byte, shift = 2 + sub // 2, 4 * (sub % 2)
        old = int(b2[byte])
        sc = (old >> shift) & 15
        nsc = (sc + 5) % 16
        b2[byte] = ((old & (0xFF ^ (15 << shift))) | (nsc << shift)) & 0xFF
        w2 = _deq(oracle_lib, 1, b2)
        diff = np.nonzero(w2 != base)[0]
        assert diff.min() >= 32 * sub and diff.max() < 32 * (sub + 1)
        np.testing.assert_array_equal(w2[32 * sub:32 * sub + 32] * (2 * sc + 1), base[32 * sub:32 * sub + 32] * (2 * nsc + 1))


@pytest.mark.parametrize("seed", range(6))
def test_iq2_index_high_bit_governs_one_group(oracle_lib, seed):
    blk = _rand_block(1, seed)
    base = _deq(oracle_lib, 1, blk)
    for g in (0, 9, 22, 31):
        b2 = blk.copy()
        b2[38 + g // 8] ^= 1 << (g % 8)
        w2 = _deq(oracle_lib, 1, b2)
        diff = np.nonzero(w2 != base)[0]
        assert set(diff.tolist()) <= set(range(8 * g, 8 * g + 8)) and len(diff) > 0


@pytest.mark.parametrize("seed", range(4))
def test_iq2_d_scales_all(oracle_lib, seed):
    blk = _rand_block(1, seed)
    base = _deq(oracle_lib, 1, blk)
    b2 = blk.copy()
    d = int(b2[0]) | (int(b2[1]) << 8)
    d += 1 << 10  # exponent + 1: doubles d
    b2[0], b2[1] = d & 0xFF, d >> 8
    np.testing.assert_array_equal(_deq(oracle_lib, 1, b2), 2 * base)


@pytest.mark.parametrize("seed", range(6))
def test_iq1_delta_bit(oracle_lib, seed):
    blk = _rand_block(2, seed)
    base = _deq(oracle_lib, 2, blk)
    field = sum(int(blk[50 + i]) << (8 * i) for i in range(6))
    d = float(np.array([int(blk[0]) | (int(blk[1]) << 8)], np.uint16).view(np.float16)[0])
    for g in (0, 1, 14, 31):
        b2 = blk.copy()
        b2[34 + g // 2] ^= 8 << (4 * (g % 2))
        w2 = _deq(oracle_lib, 2, b2)
        diff = np.nonzero(w2 != base)[0]
        assert diff.tolist() == list(range(8 * g, 8 * g + 8))
        sc = (field >> (3 * (g // 2))) & 7
        step = np.abs(w2[8 * g:8 * g + 8] - base[8 * g:8 * g + 8])
        np.testing.assert_array_equal(step, np.full(8, d * (2 * sc + 1) * 0.25))


@pytest.mark.parametrize("seed", range(6))
def test_iq1_subscale_governs_16_weights(oracle_lib, seed):
    blk = _rand_block(2, seed)
    base = _deq(oracle_lib, 2, blk)
    field = sum(int(blk[50 + i]) << (8 * i) for i in range(6))
    for sub in range(16):
        sc = (field >> (3 * sub)) & 7
        nsc = (sc + 3) % 8
        f2 = (field & ~(7 << (3 * sub))) | (nsc << (3 * sub))
        b2 = blk.copy()
        for i in range(6):
            b2[50 + i] = (f2 >> (8 * i)) & 0xFF
        w2 = _deq(oracle_lib, 2, b2)
        diff = np.nonzero(w2 != base)[0]
        assert len(diff) == 0 or (diff.min() >= 16 * sub and diff.max() < 16 * (sub + 1))
        np.testing.assert_array_equal(w2[16 * sub:16 * sub + 16] * (2 * sc + 1), base[16 * sub:16 * sub + 16] * (2 * nsc + 1))


@pytest.mark.parametrize("seed", range(6))
def test_iq1_index_high_bits_govern_one_group(oracle_lib, seed):
    blk = _rand_block(2, seed)
    base = _deq(oracle_lib, 2, blk)
    for g in (0, 5, 20, 31):
        for bit in range(3):
            b2 = blk.copy()
            b2[34 + g // 2] ^= (1 << bit) << (4 * (g % 2))
            w2 = _deq(oracle_lib, 2, b2)
            diff = np.nonzero(w2 != base)[0]
            assert set(diff.tolist()) <= set(range(8 * g, 8 * g + 8)) and len(diff) > 0


def test_multi_row_block_sharing(oracle_lib):
    """k < 256: one block spans 256/k rows; row r, column c is weight r*k + c of the sequence."""
    g2, _ = _grids()
    grid = oracle_lib.expand_grid(1, g2)
    m = fixtures.make_matrix(5, 1, 256, 64, 3)
    full = oracle_lib.dequant_matrix(1, m, 256, 64, grid)
    flat = oracle_lib.dequant_matrix(1, m, 1, 256 * 64, grid)[0]
    np.testing.assert_array_equal(full.reshape(-1), flat)
    blk0 = oracle_lib.dequant_matrix(1, m[:74], 1, 256, grid)[0]
    np.testing.assert_array_equal(full[:4].reshape(-1), blk0)


def test_dequant_values_exact_in_fp32(oracle_lib):
    w = fixtures.workload(2)
    for q, g in ((1, w.grid_iq2), (2, w.grid_iq1)):
        grid = oracle_lib.expand_grid(q, g)
        m = fixtures.make_matrix(11, q, 64, 2048, 0)
        d = oracle_lib.dequant_matrix(q, m, 64, 2048, grid)
        assert np.array_equal(d.astype(np.float32).astype(np.float64), d)
        rms = np.sqrt((d ** 2).mean())
        assert 0.005 < rms < 0.08  # |W| ~ 1/sqrt(2048) keeps activations O(1)
