"""Pins of the oracle's routed layer.

- closed form: experts whose every weight is one constant give
  out = sum_k w_k * c_d * F * silu(c_g * S) * c_u * S, S = sum(x)
  (Red Metal dev8, steps 4-5: gate, up, SiLU(gate)*up, down, then
  accumulator += router_weight * expert_output);
- an independent numpy restatement (dense matrices, matrix products) on small
  configs, which catches a transposed operand or a wrong index;
- invariants: linearity in the router weights, order of the k slots, zero
  weights, aliased ids, bad ids contributing nothing."""
import math

import numpy as np
import pytest

import fixtures

H, F, E = 256, 64, 8


def _const_matrix(qtype, rows, k, d_bits, sc):
    nblk = rows * k // 256
    if qtype == 1:
        blk = np.zeros(74, np.uint8)
        blk[0], blk[1] = d_bits & 0xFF, d_bits >> 8
        blk[2:6] = sc | (sc << 4)
    else:
        blk = np.zeros(56, np.uint8)
        blk[0], blk[1] = d_bits & 0xFF, d_bits >> 8
        field = 0
        for b in range(16):
            field |= sc << (3 * b)
        for i in range(6):
            blk[50 + i] = (field >> (8 * i)) & 0xFF
    return np.tile(blk, nblk)


def _fp16(bits):
    return float(np.array([bits], np.uint16).view(np.float16)[0])


def _const_value(qtype, d_bits, sc):
    # IQ2: grid entry 0 is all symbol 1 (value 25), sign +;  IQ1: entry 0 all symbol 2 (+1), delta +1/8.
    return _fp16(d_bits) * (2 * sc + 1) / 8 * 25 if qtype == 1 else _fp16(d_bits) * (2 * sc + 1) * 1.125


def _grids(oracle_lib):
    g2 = np.zeros(512, np.uint16)
    g2[0] = 0x5555
    g1 = np.zeros(2048, np.uint16)
    g1[0] = 0xAAAA
    return oracle_lib.expand_grid(1, g2), oracle_lib.expand_grid(2, g1)


@pytest.mark.parametrize("qtype", [1, 2])
def test_closed_form_constant_experts(oracle_lib, qtype):
    g2, g1 = _grids(oracle_lib)
    params = [(0x1400, 3, 0x1500, 5, 0x1000, 1), (0x1800, 0, 0x1200, 7, 0x1700, 2)]
    if qtype == 2:
        params = [(0x1C00, 2, 0x1D00, 1, 0x1800, 3), (0x2000, 0, 0x1E00, 4, 0x1B00, 6)]
    experts, consts = [], []
    for dg, sg, du, su, dd, sd in params:
        ex = fixtures.Expert(qtype, F, _const_matrix(qtype, F, H, dg, sg), _const_matrix(qtype, F, H, du, su),
                             _const_matrix(qtype, H, F, dd, sd))
        experts.append(ex)
        consts.append((_const_value(qtype, dg, sg), _const_value(qtype, du, su), _const_value(qtype, dd, sd)))
    x = fixtures.make_x(3, 2, H)
    ids = np.array([[0, 1], [1, 1]], np.int32)
    w = np.array([[0.25, 0.75], [0.5, 1.5]], np.float32)
    out = oracle_lib.moe_layer(x, ids, w, experts, grid_iq2=g2, grid_iq1=g1)
    for t in range(2):
        S = float(np.sum(x[t].astype(np.float64)))
        want = 0.0
        for s in range(2):
            cg, cu, cd = consts[ids[t, s]]
            g = cg * S
            want += float(w[t, s]) * cd * F * (g / (1.0 + math.exp(-g))) * (cu * S)
        np.testing.assert_allclose(out[t], np.full(H, want), rtol=1e-12, atol=0)


def _small_problem(oracle_lib, mixed=True, seed=21):
    w = fixtures.workload(1)
    qts = [1 if (e % 2 == 0 or not mixed) else 2 for e in range(E)]
    experts = [fixtures.make_expert(seed, qts[e], H, F, e) for e in range(E)]
    shared = fixtures.make_expert(seed, 2 if mixed else 1, H, 2 * F, 99)
    g2 = oracle_lib.expand_grid(1, w.grid_iq2)
    g1 = oracle_lib.expand_grid(2, w.grid_iq1)
    x = fixtures.make_x(seed, 5, H)
    st = fixtures.Stream(seed, 8)
    ids = st.randint(5 * 3, E).astype(np.int32).reshape(5, 3)
    wt = (0.2 + st.uniform(15)).astype(np.float32).reshape(5, 3)
    return experts, shared, g2, g1, x, ids, wt


def _numpy_dense(oracle_lib, experts, shared, g2, g1, x, ids, wt):
    def dense(ex):
        grid = g2 if ex.qtype == 1 else g1
        Wg = oracle_lib.dequant_matrix(ex.qtype, ex.gate, ex.ffn, H, grid)
        Wu = oracle_lib.dequant_matrix(ex.qtype, ex.up, ex.ffn, H, grid)
        Wd = oracle_lib.dequant_matrix(ex.qtype, ex.down, H, ex.ffn, grid)
        return Wg, Wu, Wd

    X = x.astype(np.float64)
    out = np.zeros((x.shape[0], H))
    for e in sorted(set(ids.reshape(-1).tolist())):
        Wg, Wu, Wd = dense(experts[e])
        G, U = X @ Wg.T, X @ Wu.T
        Y = (G * (1.0 / (1.0 + np.exp(-G))) * U) @ Wd.T
        coef = np.where(ids == e, wt.astype(np.float64), 0.0).sum(axis=1)
        out += coef[:, None] * Y
    if shared is not None:
        Wg, Wu, Wd = dense(shared)
        G, U = X @ Wg.T, X @ Wu.T
        out += (G * (1.0 / (1.0 + np.exp(-G))) * U) @ Wd.T
    return out


@pytest.mark.parametrize("mixed", [False, True])
def test_numpy_dense_restatement(oracle_lib, mixed):
    experts, shared, g2, g1, x, ids, wt = _small_problem(oracle_lib, mixed)
    got = oracle_lib.moe_layer(x, ids, wt, experts, shared, g2, g1)
    want = _numpy_dense(oracle_lib, experts, shared, g2, g1, x, ids, wt)
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-13)


def test_numpy_dense_restatement_tiny_workload(oracle_lib):
    w = fixtures.workload(1)
    got = oracle_lib.workload_layer(w)
    experts = [w.expert(e) for e in range(w.n_experts)]
    want = _numpy_dense(oracle_lib, experts, None, oracle_lib.expand_grid(1, w.grid_iq2),
                        oracle_lib.expand_grid(2, w.grid_iq1), w.x, w.ids, w.weights)
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-13)


def test_linearity_in_router_weights(oracle_lib):
    experts, _, g2, g1, x, ids, wt = _small_problem(oracle_lib)
    L = lambda ww: oracle_lib.moe_layer(x, ids, ww, experts, None, g2, g1)
    wt = (np.round(wt * 1024) / 1024).astype(np.float32)  # dyadic: fp32 sums below are exact
    base = L(wt)
    np.testing.assert_allclose(L(wt * np.float32(2.0)), 2.0 * base, rtol=1e-13, atol=1e-15)
    w2 = (wt[:, ::-1] * np.float32(0.5)).copy()
    np.testing.assert_allclose(L(wt + w2), base + L(w2), rtol=1e-10, atol=1e-12)


def test_slot_order_invariance(oracle_lib):
    experts, shared, g2, g1, x, ids, wt = _small_problem(oracle_lib)
    base = oracle_lib.moe_layer(x, ids, wt, experts, shared, g2, g1)
    perm = [2, 0, 1]
    np.testing.assert_allclose(oracle_lib.moe_layer(x, ids[:, perm], wt[:, perm], experts, shared, g2, g1), base,
                               rtol=1e-12, atol=1e-14)


def test_zero_weight_contributes_nothing(oracle_lib):
    experts, _, g2, g1, x, ids, wt = _small_problem(oracle_lib)
    w0 = wt.copy()
    w0[:, 1] = 0.0
    a = oracle_lib.moe_layer(x, ids, w0, experts, None, g2, g1)
    b = oracle_lib.moe_layer(x, ids[:, [0, 2]], wt[:, [0, 2]], experts, None, g2, g1)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-15)


def test_identical_experts_normalised_equal_single(oracle_lib):
    experts, _, g2, g1, x, _, _ = _small_problem(oracle_lib)
    copies = [experts[3]] + [fixtures.Expert(experts[3].qtype, F, experts[3].gate.copy(), experts[3].up.copy(),
                                             experts[3].down.copy()) for _ in range(3)]
    ids = np.tile(np.array([[0, 1, 2, 3]], np.int32), (x.shape[0], 1))
    wt = np.tile(np.array([[0.125, 0.25, 0.375, 0.25]], np.float32), (x.shape[0], 1))
    many = oracle_lib.moe_layer(x, ids, wt, copies, None, g2, g1)
    one = oracle_lib.moe_layer(x, np.zeros((x.shape[0], 1), np.int32), np.ones((x.shape[0], 1), np.float32),
                               copies, None, g2, g1)
    np.testing.assert_allclose(many, one, rtol=1e-12, atol=1e-14)
    alias = oracle_lib.moe_layer(x, np.zeros((x.shape[0], 4), np.int32), wt, copies, None, g2, g1)
    np.testing.assert_allclose(alias, one, rtol=1e-12, atol=1e-14)


def test_bad_ids_contribute_nothing(oracle_lib):
    experts, _, g2, g1, x, ids, wt = _small_problem(oracle_lib)
    bad = ids.copy()
    bad[0, 1] = E + 3
    bad[2, 0] = -1
    out, rc = oracle_lib.moe_layer(x, bad, wt, experts, None, g2, g1, return_rc=True)
    assert rc == oracle_lib.SKIPPED_PAIRS
    w0 = wt.copy()
    w0[0, 1] = 0.0
    w0[2, 0] = 0.0
    ref = oracle_lib.moe_layer(x, np.where(bad < 0, 0, np.where(bad >= E, 0, bad)), w0, experts, None, g2, g1)
    np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-15)


def test_missing_expert_contributes_nothing(oracle_lib):
    experts, _, g2, g1, x, ids, wt = _small_problem(oracle_lib)
    ex = list(experts)
    victim = int(ids[1, 0])
    ex[victim] = None
    out, rc = oracle_lib.moe_layer(x, ids, wt, ex, None, g2, g1, return_rc=True)
    assert rc == oracle_lib.SKIPPED_PAIRS
    w0 = np.where(ids == victim, 0.0, wt).astype(np.float32)
    ref = oracle_lib.moe_layer(x, ids, w0, experts, None, g2, g1)
    np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-15)


def test_zero_tokens_is_noop(oracle_lib):
    experts, _, g2, g1, _, _, _ = _small_problem(oracle_lib)
    out = oracle_lib.moe_layer(np.zeros((0, H), np.float32), np.zeros((0, 2), np.int32), np.zeros((0, 2), np.float32),
                               experts, None, g2, g1, hidden=H)
    assert out.shape == (0, H)


def test_threads_do_not_change_result(oracle_lib):
    experts, shared, g2, g1, x, ids, wt = _small_problem(oracle_lib)
    n0 = oracle_lib.set_threads(0)
    a = oracle_lib.moe_layer(x, ids, wt, experts, shared, g2, g1)
    oracle_lib.set_threads(1)
    b = oracle_lib.moe_layer(x, ids, wt, experts, shared, g2, g1)
    oracle_lib.set_threads(n0)
    np.testing.assert_array_equal(a, b)
