"""Pins of the oracle's codebook expansion and scalar conversions.

Grid values are pinned to hand-worked examples (tests/golden/grid_examples.json,
Red Lite dev10, section 'Quant grids'); fp16 decoding and bf16 rounding are
pinned to numpy's and torch's own conversions, which share no code with the
oracle."""
import json
import os

import numpy as np
import pytest
import torch

import fixtures

GOLD = os.path.join(os.path.dirname(__file__), "golden", "grid_examples.json")


def _gold():
    with open(GOLD) as f:
        return json.load(f)


@pytest.mark.parametrize("fmt,qtype", [("iq2", 1), ("iq1", 2)])
def test_grid_golden(oracle_lib, fmt, qtype):
    g = _gold()
    compact = np.array([int(e["compact"], 16) for e in g[fmt]], np.uint16)
    out = oracle_lib.expand_grid(qtype, compact).reshape(-1, 8)
    want = np.array([e["values"] for e in g[fmt]], np.int8)
    np.testing.assert_array_equal(out, want)


@pytest.mark.parametrize("qtype", [1, 2])
def test_grid_symbol3_rejected(oracle_lib, qtype):
    for c in _gold()["invalid"]:
        assert oracle_lib.expand_grid_rc(qtype, np.array([0x5555, int(c, 16)], np.uint16)) == oracle_lib.EINVAL


def test_grid_bad_qtype(oracle_lib):
    assert oracle_lib.expand_grid_rc(7, np.array([0], np.uint16)) == oracle_lib.EINVAL


@pytest.mark.parametrize("qtype", [1, 2])
def test_grid_all_patterns_bijective(oracle_lib, qtype):
    """All 3^8 valid compact codes expand to 3^8 distinct value patterns over the
    three-value alphabet, each value position independently taking all three values."""
    codes = []
    for p in range(6561):
        c, q = 0, p
        for j in range(8):
            c |= (q % 3) << (2 * j)
            q //= 3
        codes.append(c)
    out = oracle_lib.expand_grid(qtype, np.array(codes, np.uint16)).reshape(-1, 8)
    alphabet = {1: {8, 25, 43}, 2: {-1, 0, 1}}[qtype]
    assert set(np.unique(out).tolist()) == alphabet
    assert len({bytes(r) for r in out.astype(np.int8)}) == 6561
    for j in range(8):
        vals, cnt = np.unique(out[:, j], return_counts=True)
        assert cnt.tolist() == [2187, 2187, 2187]


def test_seeded_grids_valid(oracle_lib):
    for cfg in (1, 2):
        w = fixtures.workload(cfg)
        for qtype, g in ((1, w.grid_iq2), (2, w.grid_iq1)):
            assert len(set(g.tolist())) == g.size  # distinct entries
            oracle_lib.expand_grid(qtype, g)  # no symbol 3


FP16_CASES = [0x0000, 0x8000, 0x0001, 0x03FF, 0x0400, 0x3C00, 0x3C01, 0x3555, 0x7BFF, 0xFBFF, 0xC000, 0x7C00, 0xFC00,
              0x1000, 0x1FFF, 0x2400]


def test_fp16_decode_matches_numpy(oracle_lib):
    for h in FP16_CASES + list(range(0, 0x7C00, 97)):
        want = float(np.array([h], np.uint16).view(np.float16)[0])
        assert oracle_lib.fp16_to_double(h) == want, hex(h)


def test_fp16_nan(oracle_lib):
    assert np.isnan(oracle_lib.fp16_to_double(0x7E00))


def test_bf16_rne_matches_torch(oracle_lib):
    st = fixtures.Stream(123, 9)
    bits = st.u64(4000).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    ties = np.array([0x3F808000, 0x3F818000, 0xBF808000, 0x3F80FFFF, 0x3F807FFF, 0x7F7FFFFF, 0x00008000, 0x00018000],
                    np.uint32).view(np.float32)
    f = np.concatenate([f, ties, np.array([1.0, -2.5, 3.0e38, 1e-40], np.float32)])
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle_lib.float_to_bf16(f)
    np.testing.assert_array_equal(got, want)


def test_shape_rule(oracle_lib):
    assert oracle_lib.shape_ok(512, 2048)
    assert oracle_lib.shape_ok(2048, 512)
    assert oracle_lib.shape_ok(256, 64)  # block spans 4 rows
    assert not oracle_lib.shape_ok(256, 48)  # 48 does not divide 256
    assert not oracle_lib.shape_ok(256, 16)  # groups would be fine, sub-blocks of 32 would straddle
    assert not oracle_lib.shape_ok(3, 64)  # 192 weights: not whole blocks
    assert not oracle_lib.shape_ok(1, 300)
