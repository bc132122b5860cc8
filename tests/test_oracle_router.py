"""Pins of the oracle's router (softmax, top-k, renormalisation) and of the
block around the layer (RMSNorm, router, layer, residual).

Router: hand-worked golden cases (tests/golden/router_examples.json, closed
forms), the numpy input recipe that drew the batched-decode workload's
routing, brute force over every k-subset on small cases, and invariants
(shift of the logits, permutation of the experts).  Block: special cases
with closed forms (constant hidden states, constant experts, all-zero
experts) and RMSNorm's scale invariance."""
import itertools
import json
import math
import os

import numpy as np
import pytest

import fixtures

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "router_examples.json")


def test_router_golden_examples(oracle_lib):
    for ex in json.load(open(GOLDEN))["examples"]:
        ids, w = oracle_lib.route_topk(np.array([ex["logits"]], np.float32), ex["k"])
        assert ids[0].tolist() == ex["ids"], ex["why"]
        np.testing.assert_allclose(w[0], ex["weights"], rtol=1e-14, atol=0, err_msg=ex["why"])


def test_router_matches_the_workload_recipe(oracle_lib):
    """The batched-decode workload's routing was drawn by a numpy restatement
    (fixtures.softmax_topk_routing): same ids, weights to fp32 rounding."""
    st = fixtures.Stream(fixtures.SEED_BASE + 4, 4)
    logits = st.normal(64 * 512).reshape(64, 512).astype(np.float32)
    ids, w = oracle_lib.route_topk(logits, 10)
    want_ids, want_w = fixtures.softmax_topk_routing(logits.astype(np.float64), 10)
    assert np.array_equal(ids, want_ids)
    np.testing.assert_allclose(w, want_w, rtol=1e-6)
    w4 = fixtures.workload(4)
    assert np.array_equal(ids, w4.ids)


@pytest.mark.parametrize("E,k", [(6, 3), (7, 1), (5, 5)])
def test_router_brute_force(oracle_lib, E, k):
    """On small cases the chosen k experts have the largest total probability
    of all k-subsets, come in descending order, and their weights sum to 1."""
    st = fixtures.Stream(17, E, k)
    logits = (st.normal(20 * E) * 2.0).reshape(20, E).astype(np.float32)
    ids, w = oracle_lib.route_topk(logits, k)
    for t in range(20):
        p = np.exp(logits[t].astype(np.float64) - logits[t].max())
        p /= p.sum()
        best = max(itertools.combinations(range(E), k), key=lambda c: (sum(p[list(c)]), [-i for i in c]))
        assert sorted(ids[t].tolist()) == sorted(best)
        assert all(p[ids[t][j]] >= p[ids[t][j + 1]] for j in range(k - 1))
        assert abs(w[t].sum() - 1.0) < 1e-14


def test_router_invariants(oracle_lib):
    st = fixtures.Stream(23, 1)
    logits = st.normal(8 * 40).reshape(8, 40).astype(np.float32)
    ids, w = oracle_lib.route_topk(logits, 6)
    # adding a constant (exactly representable shift) changes nothing
    ids2, w2 = oracle_lib.route_topk(logits + np.float32(4.0), 6)
    assert np.array_equal(ids, ids2)
    np.testing.assert_allclose(w, w2, rtol=1e-6)
    # relabelling the experts relabels the choice
    perm = np.argsort(st.uniform(40))
    ids3, w3 = oracle_lib.route_topk(logits[:, perm], 6)
    assert np.array_equal(perm[ids3], ids)
    np.testing.assert_allclose(w3, w, rtol=1e-15)


def test_router_rejects(oracle_lib):
    lg = np.zeros((1, 4), np.float32)
    with pytest.raises(ValueError):
        oracle_lib.route_topk(lg, 5)
    with pytest.raises(ValueError):
        oracle_lib.route_topk(lg, 0)


# ------------------------------------------------------------------ block

H, F, E = 256, 64, 6


def _const_matrix(qtype, rows, k, d_bits, sc):
    nblk = rows * k // 256
    blk = np.zeros(74, np.uint8)
    blk[0], blk[1] = d_bits & 0xFF, d_bits >> 8
    blk[2:6] = sc | (sc << 4)
    return np.tile(blk, nblk)


def _const_expert(dg, dd):
    """IQ2_XS-style expert whose gate/up weights all equal c_g and down weights c_d
    (grid entry 0 = all symbol 1 -> 25, sub-scale 0 -> (2*0+1)/8, sign +)."""
    return fixtures.Expert(1, F, _const_matrix(1, F, H, dg, 0), _const_matrix(1, F, H, dg, 0),
                           _const_matrix(1, H, F, dd, 0))


def _fp16(bits):
    return float(np.array([bits], np.uint16).view(np.float16)[0])


def _grids(oracle_lib):
    g2 = np.zeros(512, np.uint16)
    g2[0] = 0x5555
    return oracle_lib.expand_grid(1, g2), oracle_lib.expand_grid(2, np.zeros(2048, np.uint16))


def test_block_closed_form(oracle_lib):
    """h = c * ones, gamma = ones, eps = 3, c = 1: RMSNorm gives xn = 1/2 everywhere
    (mean of squares, not sum), S = sum(xn) = H/2.  Router rows alpha_e * ones give
    logits alpha_e * S; constant experts give y = c_d * F * silu(c_g S) * c_g S per
    row; out = h + sum_k w_k y_k."""
    g2, g1 = _grids(oracle_lib)
    dgs = [0x1000, 0x1100, 0x1200, 0x1300, 0x1400, 0x1500]
    experts = [_const_expert(dg, 0x1400 + 0x40 * e) for e, dg in enumerate(dgs)]
    alpha = np.array([0.001, 0.004, -0.002, 0.003, 0.0, 0.002], np.float32)
    router = np.repeat(alpha[:, None], H, axis=1)
    h = np.ones((1, H), np.float32)
    gamma = np.ones(H, np.float32)
    out, ids, w = oracle_lib.moe_block(h, gamma, 3.0, router, 3, experts, grid_iq2=g2, grid_iq1=g1,
                                       return_routing=True)
    S = H / 2.0
    lg = alpha.astype(np.float64) * S
    assert ids[0].tolist() == [1, 3, 5]  # alpha 0.004, 0.003, 0.002 (ids 2 < 5 lose: alpha[2] < 0)
    sel = np.exp(lg[[1, 3, 5]] - lg.max())
    want_w = sel / sel.sum()
    np.testing.assert_allclose(w[0], want_w, rtol=1e-14)
    y = 0.0
    for j, e in enumerate([1, 3, 5]):
        cg = _fp16(dgs[e]) / 8 * 25
        cd = _fp16(0x1400 + 0x40 * e) / 8 * 25
        g = cg * S
        y += want_w[j] * cd * F * (g / (1.0 + math.exp(-g))) * g
    np.testing.assert_allclose(out[0], 1.0 + y, rtol=1e-12)


def test_block_zero_experts_is_the_residual(oracle_lib):
    """Experts whose block scale d is 0 have all weights 0: out = h exactly."""
    g2, g1 = _grids(oracle_lib)
    experts = [_const_expert(0x0000, 0x0000) for _ in range(E)]
    h = fixtures.make_x(5, 3, H)
    st = fixtures.Stream(5, 9)
    router = st.normal(E * H).reshape(E, H).astype(np.float32)
    gamma = (1.0 + 0.1 * st.normal(H)).astype(np.float32)
    out = oracle_lib.moe_block(h, gamma, 1e-6, router, 2, experts, shared=experts[0], grid_iq2=g2, grid_iq1=g1)
    assert np.array_equal(out, h.astype(np.float64))


def test_block_scale_invariance_and_layer_composition(oracle_lib):
    """With eps = 0, RMSNorm(a h) = RMSNorm(h), so block(a h) - a h = block(h) - h;
    and block(h) - h equals the layer oracle run on the normalised state with
    the block's own routing."""
    w = fixtures.workload(1)
    experts = [w.expert(e) for e in range(w.n_experts)]
    g2 = oracle_lib.expand_grid(1, w.grid_iq2)
    g1 = oracle_lib.expand_grid(2, w.grid_iq1)
    st = fixtures.Stream(11, 2)
    h = fixtures.make_x(11, 4, w.hidden)
    gamma = (1.0 + 0.1 * st.normal(w.hidden)).astype(np.float32)
    router = (0.05 * st.normal(w.n_experts * w.hidden)).reshape(w.n_experts, w.hidden).astype(np.float32)
    out, ids, wt = oracle_lib.moe_block(h, gamma, 0.0, router, 4, experts, grid_iq2=g2, grid_iq1=g1,
                                        return_routing=True)
    out2 = oracle_lib.moe_block(h * np.float32(4.0), gamma, 0.0, router, 4, experts, grid_iq2=g2, grid_iq1=g1)
    np.testing.assert_allclose(out2 - 4.0 * h, out - h, rtol=1e-9, atol=1e-12 * np.abs(out - h).max())
    hd = h.astype(np.float64)
    xn = gamma * hd / np.sqrt((hd * hd).mean(axis=1, keepdims=True))
    lay = oracle_lib.moe_layer(xn.astype(np.float32), ids, wt.astype(np.float32), experts, grid_iq2=g2, grid_iq1=g1)
    np.testing.assert_allclose(out - h, lay, rtol=0, atol=1e-5 * np.abs(lay).max())
