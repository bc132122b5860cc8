"""The router kernel (softmax, top-k, renormalisation) and the block around
the layer (RMSNorm, router, layer, residual) against the fp64 oracle.

Router: expert ids bit-exact (the kernel ranks on the logits, the oracle on
fp64 probabilities: the same order for the finite, non-underflowing logits
drawn here), weights within 1e-6 relative.  Block: inputs drawn so that the
top-k choice has a clear margin (the kernel's fp32 logits cannot flip it),
then out within 1e-4 of the MoE part's max |value| on the fp32-accumulate
path and 2e-2 on the bf16 tensor-core path."""
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


def _route(P, logits, k):
    lg = torch.from_numpy(np.ascontiguousarray(logits, np.float32)).cuda()
    T, E = logits.shape
    ids = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), float("nan"), dtype=torch.float32, device="cuda")
    assert P.redlite_moe_route_topk(lg, T, E, k, ids, w) == P.REDLITE_OK
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy().astype(np.float64)


def test_router_on_the_batched_workload_logits(P, oracle_lib):
    st = fixtures.Stream(fixtures.SEED_BASE + 4, 4)
    logits = st.normal(64 * 512).reshape(64, 512).astype(np.float32)
    ids, w = _route(P, logits, 10)
    want_ids, want_w = oracle_lib.route_topk(logits, 10)
    assert np.array_equal(ids, want_ids)
    assert np.array_equal(ids, fixtures.workload(4).ids)
    assert np.abs(w - want_w).max() <= 1e-6 * np.abs(want_w).max()


@pytest.mark.parametrize("T,E,k", [(1, 16, 4), (7, 100, 1), (300, 512, 16), (33, 1000, 10), (5, 1024, 16),
                                   (3, 16, 16), (9, 513, 7)])
def test_router_shapes(P, oracle_lib, T, E, k):
    st = fixtures.Stream(31337, T, E, k)
    logits = (3.0 * st.normal(T * E)).reshape(T, E).astype(np.float32)
    ids, w = _route(P, logits, k)
    want_ids, want_w = oracle_lib.route_topk(logits, k)
    assert np.array_equal(ids, want_ids)
    np.testing.assert_allclose(w, want_w, rtol=1e-6, atol=0)


def test_router_ties_go_to_the_lower_id(P, oracle_lib):
    """Logits from a set of five values: most experts tie with others; the
    choice and its order must be the oracle's (lower id first)."""
    st = fixtures.Stream(4711, 3)
    vals = np.array([-1.0, 0.0, 0.5, 1.5, 2.0], np.float32)
    logits = vals[st.randint(40 * 300, 5)].reshape(40, 300)
    ids, w = _route(P, logits, 12)
    want_ids, want_w = oracle_lib.route_topk(logits, 12)
    assert np.array_equal(ids, want_ids)
    np.testing.assert_allclose(w, want_w, rtol=1e-6, atol=0)


# ------------------------------------------------------------------ block


def _block_case(oracle_lib, seed, T, H=512, E=64, F=256, k=4, shared=True):
    # the first seed from `seed` on whose inputs every token's k-th and
    # (k+1)-th logit differ by more than 1e-4 (a margin the kernel's fp32
    # logits cannot cross), so the routing is unique
    for s in range(seed, seed + 100):
        st = fixtures.Stream(s, 1)
        h = fixtures.make_x(s, T, H)
        gamma = (1.0 + 0.1 * st.normal(H)).astype(np.float32)
        router = (0.05 * st.normal(E * H)).reshape(E, H).astype(np.float32)
        hd = h.astype(np.float64)
        xn = gamma * hd / np.sqrt((hd * hd).mean(axis=1, keepdims=True) + 1e-6)
        lg = np.sort(xn @ router.T.astype(np.float64), axis=1)[:, ::-1]
        if (lg[:, k - 1] - lg[:, k]).min() > 1e-4:
            break
    else:
        raise AssertionError("no seed with a clear routing margin")
    g2, g1 = fixtures.make_grid(seed, 1), fixtures.make_grid(seed, 2)
    experts = [fixtures.make_expert(seed, 1 + (e % 2), H, F, e) for e in range(E)]
    sh = fixtures.make_expert(seed, 1, H, F, 999) if shared else None
    ref = oracle_lib.moe_block(h, gamma, 1e-6, router, k, experts, sh, oracle_lib.expand_grid(1, g2),
                               oracle_lib.expand_grid(2, g1))
    return dict(H=H, E=E, F=F, k=k, T=T, g2=g2, g1=g1, experts=experts, sh=sh, h=h, gamma=gamma, router=router,
                ref=ref)


def _run_block(P, c, in_place=False, general=False):
    L = P.MoeLayer(c["H"], c["E"], c["F"], c["T"], c["k"], c["g2"], c["g1"],
                   pool_bytes=(c["E"] + 2) * fixtures.expert_bytes(1, c["H"], c["F"]) + 4096)
    assert L.upload(list(range(c["E"])), c["experts"]) == 0
    if c["sh"] is not None:
        assert L.set_shared(c["sh"]) == 0
    if general:
        L.table.min_ffn = 0
    h = torch.from_numpy(c["h"]).cuda()
    gamma = torch.from_numpy(c["gamma"]).cuda()
    router = torch.from_numpy(c["router"]).cuda()
    scratch = torch.zeros(P.redlite_moe_block_scratch_bytes(c["H"], c["E"], c["T"], c["k"]), dtype=torch.uint8,
                          device="cuda")
    out = h.clone() if in_place else torch.full_like(h, float("nan"))
    rc = P.redlite_moe_block(out if in_place else h, c["T"], gamma, 1e-6, router, c["k"], L.table, L.shared, out,
                             scratch)
    torch.cuda.synchronize()
    assert rc == P.REDLITE_OK
    assert L.read_status() == 0
    return out.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("T", [1, 8, 20])
def test_block_matches_oracle(P, oracle_lib, T):
    c = _block_case(oracle_lib, 600 + T, T)
    got = _run_block(P, c)
    moe = c["ref"] - c["h"]
    assert np.abs(got - c["ref"]).max() <= 1e-4 * np.abs(moe).max()


def test_block_in_place_and_general_path(P, oracle_lib):
    c = _block_case(oracle_lib, 777, 6)
    moe = c["ref"] - c["h"]
    got = _run_block(P, c, in_place=True)
    assert np.abs(got - c["ref"]).max() <= 1e-4 * np.abs(moe).max()
    got = _run_block(P, c, general=True)  # CUDA-core tiles (out starts from the residual by a copy)
    assert np.abs(got - c["ref"]).max() <= 1e-4 * np.abs(moe).max()


def test_block_tensor_core_path(P, oracle_lib):
    """200 tokens x top-4 (800 pairs): the bucketed tcgen05 path under the block."""
    c = _block_case(oracle_lib, 888, 200)
    got = _run_block(P, c)
    moe = c["ref"] - c["h"]
    assert np.abs(got - c["ref"]).max() <= 2e-2 * np.abs(moe).max()
