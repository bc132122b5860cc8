"""Layer parity of the CUDA path against the fp64 oracle on the seeded
workloads, plus invariants and device-side error reporting.

Tolerance: max|gpu - oracle| <= tol * max|oracle| with tol = 1e-4 for the
fp32-accumulate decode path and 2e-2 for the bf16 tensor-core path."""
import numpy as np
import pytest
import torch

import fixtures
from bench import layer_for_workload

pytestmark = pytest.mark.gpu

TOL_FP32 = 1e-4
TOL_BF16 = 2e-2


@pytest.fixture(scope="module")
def P():
    from routed_expert_ffn_iq2_b200 import build

    build.build()
    import routed_expert_ffn_iq2_b200 as P

    return P


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _run(L, x, ids, wt):
    out = L(_dev(x), _dev(ids), _dev(wt))
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def _rel_err(got, ref):
    return np.abs(got - ref).max() / np.abs(ref).max()


@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_decode_workloads(P, oracle_lib, cfg):
    w = fixtures.workload(cfg)
    L = layer_for_workload(w)
    got = _run(L, w.x, w.ids, w.weights)
    ref = oracle_lib.workload_layer(w)
    assert L.read_status() == 0
    assert _rel_err(got, ref) <= TOL_FP32


def test_cold_upload_counters(P):
    """A cold top-10 selection makes 10 experts resident with 30 matrix copies."""
    w = fixtures.workload(3)
    L = layer_for_workload(w)
    assert (L.counters.loads, L.counters.copies) == (10, 30)
    assert L.counters.bytes == 10 * fixtures.expert_bytes(2, 2048, 512)


def test_batched_decode_workload(P, oracle_lib):
    w = fixtures.workload(4)
    L = layer_for_workload(w)
    got = _run(L, w.x, w.ids, w.weights)
    ref = oracle_lib.workload_layer(w)
    assert L.read_status() == 0
    assert _rel_err(got, ref) <= TOL_FP32


def test_prefill_small(P, oracle_lib):
    w = fixtures.workload(5, n_tokens=192)
    L = layer_for_workload(w)
    got = _run(L, w.x, w.ids, w.weights)
    ref = oracle_lib.workload_layer(w)
    assert L.read_status() == 0
    assert _rel_err(got, ref) <= TOL_BF16


def _prefill_rows(w):
    """Rows of the full prefill checked against the oracle: every 173rd token,
    the last token, every token of the ten rarest routed experts (their
    token tiles are partial single tiles), and 64 tokens of the hottest
    expert (which spans 29 token tiles; the pairs' order inside an expert is
    not fixed, so any of its tokens may sit in its last, partial tile)."""
    ids = w.ids
    counts = np.bincount(ids.reshape(-1), minlength=w.n_experts)
    used = np.nonzero(counts)[0]
    rare = used[np.argsort(counts[used], kind="stable")[:10]]
    hot = int(np.argmax(counts))
    hot_tokens = np.nonzero((ids == hot).any(axis=1))[0]
    rows = set(range(0, ids.shape[0], 173)) | {ids.shape[0] - 1}
    rows |= set(np.nonzero(np.isin(ids, rare).any(axis=1))[0].tolist())
    rows |= set(hot_tokens[np.linspace(0, len(hot_tokens) - 1, 64).astype(int)].tolist())
    return np.array(sorted(rows))


def test_prefill_full_sampled(P, oracle_lib):
    w = fixtures.workload(5)
    L = layer_for_workload(w)
    got = _run(L, w.x, w.ids, w.weights)
    sample = _prefill_rows(w)
    assert len(sample) >= 100
    ref = oracle_lib.workload_layer(w, tokens=sample)
    assert L.read_status() == 0
    assert _rel_err(got[sample], ref) <= TOL_BF16
    assert np.isfinite(got).all()


def test_slot_order_and_zero_weight(P):
    w = fixtures.workload(2)
    L = layer_for_workload(w)
    base = _run(L, w.x, w.ids, w.weights)
    perm = np.array([3, 9, 0, 5, 1, 8, 2, 7, 4, 6])
    permuted = _run(L, w.x, w.ids[:, perm], w.weights[:, perm])
    assert _rel_err(permuted, base) <= TOL_FP32
    w0 = w.weights.copy()
    w0[0, 4] = 0.0
    zeroed = _run(L, w.x, w.ids, w0)
    dropped = _run(L, w.x, np.delete(w.ids, 4, axis=1), np.delete(w.weights, 4, axis=1))
    assert _rel_err(zeroed, dropped) <= TOL_FP32


def test_aliased_ids_equal_single_expert(P):
    w = fixtures.workload(2)
    L = layer_for_workload(w)
    e = int(w.ids[0, 0])
    ids = np.full((1, 4), e, np.int32)
    wt = np.array([[0.125, 0.25, 0.375, 0.25]], np.float32)
    many = _run(L, w.x, ids, wt)
    one = _run(L, w.x, ids[:, :1], np.ones((1, 1), np.float32))
    assert _rel_err(many, one) <= TOL_FP32


def test_bad_ids_reported_and_skipped(P, oracle_lib):
    w = fixtures.workload(2)
    L = layer_for_workload(w)
    ids = w.ids.copy()
    ids[0, 2] = 512
    ids[0, 6] = -3
    got = _run(L, w.x, ids, w.weights)
    assert L.read_status() & P.REDLITE_STATUS_BAD_ID
    L.clear_status()
    w0 = w.weights.copy()
    w0[0, 2] = w0[0, 6] = 0
    ref = _run(L, w.x, w.ids, w0)
    assert _rel_err(got, ref) <= TOL_FP32
    assert L.read_status() == 0


def test_missing_expert_reported(P):
    w = fixtures.workload(2)
    L = layer_for_workload(w)
    ids = w.ids.copy()
    free = next(e for e in range(512) if e not in set(w.ids[0].tolist()))
    ids[0, 0] = free  # slot never uploaded: null matrices
    _run(L, w.x, ids, w.weights)
    assert L.read_status() & P.REDLITE_STATUS_BAD_EXPERT


def test_bad_and_missing_ids_on_bucketed_paths(P):
    """Invalid ids and a never-uploaded slot in a 128-token call, on the
    bucketed tensor-core path and on the general CUDA-core path: both are
    reported in the status word and their pairs contribute nothing (the same
    call with those slots' weights set to 0 agrees up to summation order)."""
    w = fixtures.workload(4)
    st = fixtures.Stream(991, 2)
    logits = st.normal(128 * 512).reshape(128, 512)
    ids, wt = fixtures.softmax_topk_routing(logits, 10)
    x = fixtures.make_x(991, 128, 2048)
    sel = sorted(set(ids.reshape(-1).tolist()))
    missing = next(e for e in range(512) if e not in set(sel))
    bad = ids.copy()
    bad[0, 2], bad[5, 7], bad[9, 0] = 512, -3, missing
    w0 = wt.copy()
    w0[0, 2] = w0[5, 7] = w0[9, 0] = 0
    L = layer_for_workload(w, experts=sel, max_tokens=128)
    for general in (False, True):
        if general:
            L.table.min_ffn = 0  # unknown widths: the general CUDA-core path runs
        got = _run(L, x, bad, wt)
        status = L.read_status()
        assert status & P.REDLITE_STATUS_BAD_ID and status & P.REDLITE_STATUS_BAD_EXPERT
        L.clear_status()
        ref = _run(L, x, ids, w0)
        assert L.read_status() == 0
        assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()


def test_max_topk_and_ragged_shapes(P, oracle_lib):
    """top_k = 16, hidden 768, ffn 128 (down rows of half a block), a shared expert of width 256,
    7 tokens (ragged against the 4-token passes)."""
    H, E, F, k, T = 768, 24, 128, 16, 7
    seed = 4242
    g2 = fixtures.make_grid(seed, 1)
    g1 = fixtures.make_grid(seed, 2)
    experts = [fixtures.make_expert(seed, 1 + (e % 2), H, F, e) for e in range(E)]
    st = fixtures.Stream(seed, 3)
    ids = st.randint(T * k, E).astype(np.int32).reshape(T, k)
    wt = (0.1 + st.uniform(T * k)).astype(np.float32).reshape(T, k)
    x = fixtures.make_x(seed, T, H)
    shared = fixtures.make_expert(seed, 2, H, 2 * F, 777)
    L = P.MoeLayer(H, E, 2 * F, T, k, g2, g1, pool_bytes=(E + 2) * fixtures.expert_bytes(1, H, 2 * F) + 4096)
    assert L.upload(list(range(E)), experts) == 0
    assert L.set_shared(shared) == 0
    got = _run(L, x, ids, wt)
    ref = oracle_lib.moe_layer(x, ids, wt, experts, shared, oracle_lib.expand_grid(1, g2),
                               oracle_lib.expand_grid(2, g1))
    assert _rel_err(got, ref) <= TOL_FP32


def test_zero_tokens_noop(P):
    w = fixtures.workload(1)
    L = layer_for_workload(w)
    out = torch.full((1, 256), 7.0, device="cuda")
    e = torch.zeros((1, 4), dtype=torch.int32, device="cuda")
    rc = P.redlite_moe_layer(out, 0, e, out, 4, L.table, None, out)
    torch.cuda.synchronize()
    assert rc == 0 and float(out[0, 0]) == 7.0


def test_repeat_calls_reuse_workspace(P):
    w = fixtures.workload(2)
    L = layer_for_workload(w)
    a = _run(L, w.x, w.ids, w.weights)
    for _ in range(3):
        b = _run(L, w.x, w.ids, w.weights)
    assert _rel_err(b, a) <= TOL_FP32


@pytest.mark.parametrize("T", [1, 3, 5, 17])
def test_batched_token_counts(P, oracle_lib, T):
    """Mixed-format batched decode with the shared expert at several token
    counts: local activation limbs (T <= 4) and the cooperative conversion."""
    w = fixtures.workload(4, n_tokens=T)
    L = layer_for_workload(w)
    got = _run(L, w.x, w.ids, w.weights)
    ref = oracle_lib.workload_layer(w)
    assert L.read_status() == 0
    assert _rel_err(got, ref) <= TOL_FP32


@pytest.mark.parametrize("T,k", [(8, 4), (11, 3)])
def test_batched_item_shape_boundary(P, oracle_lib, T, k):
    """32 (token, slot) pairs run items of one tile-block per warp, 33 pairs
    items of two; both against the oracle on the mixed-format workload with
    the shared expert (the first k slots of each token's routing)."""
    w = fixtures.workload(4, n_tokens=T)
    L = layer_for_workload(w)
    ids, wt = np.ascontiguousarray(w.ids[:, :k]), np.ascontiguousarray(w.weights[:, :k])
    got = _run(L, w.x, ids, wt)
    experts = [None] * w.n_experts
    for e in w.selected():
        experts[e] = w.expert(e)
    ref = oracle_lib.moe_layer(w.x, ids, wt, experts, w.shared(), oracle_lib.expand_grid(1, w.grid_iq2),
                               oracle_lib.expand_grid(2, w.grid_iq1))
    assert L.read_status() == 0
    assert _rel_err(got, ref) <= TOL_FP32


def test_general_path_agrees_with_fast_path(P):
    w = fixtures.workload(4, n_tokens=9)
    L = layer_for_workload(w)
    fast = _run(L, w.x, w.ids, w.weights)
    L.table.min_ffn = 0  # unknown widths: the general CUDA-core path runs
    general = _run(L, w.x, w.ids, w.weights)
    assert L.read_status() == 0
    assert _rel_err(fast, general) <= TOL_FP32


def test_tensor_core_path_mixed_formats(P, oracle_lib):
    """128 tokens x top-10 (1280 pairs): the bucketed tcgen05 path, IQ2 and IQ1
    experts and the shared expert, bf16 operands with fp32 accumulation."""
    w = fixtures.workload(4)
    st = fixtures.Stream(991, 2)
    logits = st.normal(128 * 512).reshape(128, 512)
    ids, wt = fixtures.softmax_topk_routing(logits, 10)
    x = fixtures.make_x(991, 128, 2048)
    sel = sorted(set(ids.reshape(-1).tolist()))
    L = layer_for_workload(w, experts=sel, max_tokens=128)
    got = _run(L, x, ids, wt)
    experts = [None] * 512
    for e in sel:
        experts[e] = w.expert(e)
    ref = oracle_lib.moe_layer(x, ids, wt, experts, w.shared(), oracle_lib.expand_grid(1, w.grid_iq2),
                               oracle_lib.expand_grid(2, w.grid_iq1))
    assert L.read_status() == 0
    assert _rel_err(got, ref) <= TOL_BF16


def _bf16_rne(a):
    """Round finite values to bf16 (nearest even), returned as float64."""
    u = np.asarray(a, np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def test_tensor_core_tile_boundaries(P, oracle_lib):
    """257 tokens all routed to the same three experts (top-3, one IQ2_XS-style,
    two IQ1_M-style) plus the shared expert: 771 pairs take the tcgen05 path and
    every expert's pairs span token tiles of 128, 128 and 1."""
    w = fixtures.workload(4)
    q = np.asarray(w.qtypes)
    sel = [int(np.nonzero(q == 1)[0][0]), int(np.nonzero(q == 2)[0][0]), int(np.nonzero(q == 2)[0][1])]
    T = 257
    ids = np.tile(np.array(sel, np.int32), (T, 1))
    st = fixtures.Stream(257, 4)
    wt = (st.uniform(T * 3).reshape(T, 3) + 0.1).astype(np.float32)
    x = fixtures.make_x(257, T, w.hidden)
    L = layer_for_workload(w, experts=sel, max_tokens=T)
    got = _run(L, x, ids, wt)
    experts = [None] * 512
    for e in sel:
        experts[e] = w.expert(e)
    ref = oracle_lib.moe_layer(x, ids, wt, experts, w.shared(), oracle_lib.expand_grid(1, w.grid_iq2),
                               oracle_lib.expand_grid(2, w.grid_iq1))
    assert L.read_status() == 0
    assert _rel_err(got, ref) <= TOL_BF16


def test_bf16_rounding_helper_matches_oracle(oracle_lib):
    v = fixtures.make_x(77, 4, 256).reshape(-1) * np.float32(37.0)
    want = oracle_lib.float_to_bf16(v).astype(np.uint32) << 16
    assert np.array_equal(_bf16_rne(v).astype(np.float32).view(np.uint32), want)


def test_tensor_core_path_is_repeatable(P):
    """64 calls of the tcgen05 path on the same inputs agree up to the order
    of the fp32 atomic additions into out (a few ulp): a shared-memory stage
    read before its copies landed, or refilled before its readers were done,
    shows as a large difference in some call.  (A refill racing the reads hit
    about 4% of calls, so 64 calls catch it with high probability.)
    96 tokens x top-10 over a pool of 16 experts (~60 tokens each) + shared."""
    w = fixtures.workload(4)
    q = np.asarray(w.qtypes)
    pool = [int(e) for e in np.nonzero(q == 1)[0][:8]] + [int(e) for e in np.nonzero(q == 2)[0][:8]]
    T, K = 96, 10
    st = fixtures.Stream(5150, 3)
    ids = np.zeros((T, K), np.int32)
    for t in range(T):
        ids[t] = np.array(pool)[np.argsort(st.uniform(len(pool)))[:K]]
    wt = st.uniform(T * K).reshape(T, K).astype(np.float32) + np.float32(0.05)
    wt = (wt / wt.sum(axis=1, keepdims=True)).astype(np.float32)
    x = fixtures.make_x(5150, T, w.hidden)
    L = layer_for_workload(w, experts=pool, max_tokens=T)
    outs = [_run(L, x, ids, wt) for _ in range(64)]
    assert L.read_status() == 0
    scale = np.abs(outs[0]).max()
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() <= 1e-5 * scale


def test_tensor_core_path_matches_bf16_operand_reference(P, oracle_lib):
    """72 tokens x top-10 from a pool of 12 experts (6 per format) plus the
    shared expert: the tcgen05 path against the oracle's exact weights with
    the path's own roundings applied (weights, activations and h to bf16,
    nearest even).  What remains is fp32 accumulation order and rare bf16
    ties in h, so the bar is 1e-3 of max|ref| -- tight enough that a wrong
    sub-block scale, sign or selector shows."""
    w = fixtures.workload(4)
    q = np.asarray(w.qtypes)
    pool = [int(e) for e in np.nonzero(q == 1)[0][:6]] + [int(e) for e in np.nonzero(q == 2)[0][:6]]
    T, K, H = 72, 10, w.hidden
    st = fixtures.Stream(4242, 9)
    ids = np.zeros((T, K), np.int32)
    for t in range(T):
        perm = np.argsort(st.uniform(len(pool)))
        ids[t] = np.array(pool)[perm[:K]]
    wt = st.uniform(T * K).reshape(T, K).astype(np.float32) + np.float32(0.05)
    wt = (wt / wt.sum(axis=1, keepdims=True)).astype(np.float32)
    x = fixtures.make_x(4242, T, H)
    L = layer_for_workload(w, experts=pool, max_tokens=T)
    got = _run(L, x, ids, wt)
    assert L.read_status() == 0

    grids = {1: oracle_lib.expand_grid(1, w.grid_iq2), 2: oracle_lib.expand_grid(2, w.grid_iq1)}
    xb = _bf16_rne(x)
    ref = np.zeros((T, H))

    def run_expert(ex, toks, scale):
        F = ex.ffn
        wg = _bf16_rne(oracle_lib.dequant_matrix(ex.qtype, ex.gate, F, H, grids[ex.qtype]))
        wu = _bf16_rne(oracle_lib.dequant_matrix(ex.qtype, ex.up, F, H, grids[ex.qtype]))
        wd = _bf16_rne(oracle_lib.dequant_matrix(ex.qtype, ex.down, H, F, grids[ex.qtype]))
        g = xb[toks] @ wg.T
        u = xb[toks] @ wu.T
        h = _bf16_rne(g / (1.0 + np.exp(-g)) * u)
        ref[toks] += scale[:, None] * (h @ wd.T)

    for e in pool:
        tt, kk = np.nonzero(ids == e)
        if len(tt):
            run_expert(w.expert(e), tt, wt[tt, kk].astype(np.float64))
    sh = w.shared()
    if sh is not None:
        run_expert(sh, np.arange(T), np.ones(T))
    assert _rel_err(got, ref) <= 1e-3


def test_grid_wait_gives_up_and_reports(P):
    """A grid-wide wait that can never be met (the count of CTAs that have
    initialised their part of out, which every down warp waits for, is
    corrupted from the host) gives up after its time limit, sets
    REDLITE_STATUS_TIMEOUT, and leaves the context and the workspace usable:
    the next call returns the right result with a clean status."""
    w = fixtures.workload(2)
    L = layer_for_workload(w)
    ref = _run(L, w.x, w.ids, w.weights)
    assert L.read_status() == 0
    ctrl = L.workspace.view(torch.int32)
    ctrl[5] = ctrl[6] = -(1 << 30)  # control words 5, 6: CTAs that initialised their part of out (per call parity)
    torch.cuda.synchronize()
    _run(L, w.x, w.ids, w.weights)
    assert L.read_status() & P.REDLITE_STATUS_TIMEOUT
    L.clear_status()
    again = _run(L, w.x, w.ids, w.weights)
    assert L.read_status() == 0
    assert _rel_err(again, ref) <= 1e-6


@pytest.mark.parametrize("T", [1, 200])
def test_overstated_min_ffn_is_reported_not_read(P, T):
    """A table that declares min_ffn = 256 while its slots hold width-128
    experts (interchange layout, not tiled): the fast kernels (fused decode at
    T = 1, bucketed tensor-core path at T = 200) check every selected slot,
    report REDLITE_STATUS_BAD_EXPERT and read nothing from it, so every pair
    is dropped and out is all zeros."""
    H, E, F, k = 512, 8, 128, 4
    seed = 515
    g2, g1 = fixtures.make_grid(seed, 1), fixtures.make_grid(seed, 2)
    experts = [fixtures.make_expert(seed, 1 + (e % 2), H, F, e) for e in range(E)]
    L = P.MoeLayer(H, E, 256, T, k, g2, g1, pool_bytes=(E + 1) * fixtures.expert_bytes(1, H, 256) + 4096)
    assert L.upload(list(range(E)), experts) == 0
    L.table.min_ffn = 256  # overstated: the slots are 128 wide
    st = fixtures.Stream(seed, 5)
    ids = st.randint(T * k, E).astype(np.int32).reshape(T, k)
    wt = (0.1 + st.uniform(T * k)).astype(np.float32).reshape(T, k)
    x = fixtures.make_x(seed, T, H)
    got = _run(L, x, ids, wt)
    assert L.read_status() & P.REDLITE_STATUS_BAD_EXPERT
    assert np.all(got == 0.0)


def test_alternating_call_shapes_share_one_workspace(P, oracle_lib):
    """The fused kernel keeps completion counters in the workspace between
    calls (at a fixed place, two sets alternating by call parity).  One
    workspace serves a sequence of calls that change the token count, the
    top-k, the shared expert and the path (fused decode for up to 640 pairs,
    the tensor-core path above); every call matches the fp64 oracle."""
    H, E, F, kmax, Tmax = 512, 32, 256, 6, 160
    seed = 6060
    g2, g1 = fixtures.make_grid(seed, 1), fixtures.make_grid(seed, 2)
    G2, G1 = oracle_lib.expand_grid(1, g2), oracle_lib.expand_grid(2, g1)
    experts = [fixtures.make_expert(seed, 1 + (e % 2), H, F, e) for e in range(E)]
    shared = fixtures.make_expert(seed, 1, H, F, 999)
    L = P.MoeLayer(H, E, F, Tmax, kmax, g2, g1, pool_bytes=(E + 2) * fixtures.expert_bytes(1, H, F) + 4096)
    assert L.upload(list(range(E)), experts) == 0
    assert L.set_shared(shared) == 0
    shared_desc = L.shared
    st = fixtures.Stream(seed, 7)
    # (tokens, top-k, with shared expert): the fused path up to 640 pairs
    # (kmax * Tmax = 960 > 640: the last shapes take the tensor-core path)
    for T, k, sh in [(1, 6, False), (1, 5, False), (3, 6, True), (1, 6, True), (48, 6, False),
                     (1, 2, False), (150, 6, True), (2, 6, False), (160, 6, False), (1, 6, False)]:
        ids = st.randint(T * k, E).astype(np.int32).reshape(T, k)
        wt = (0.1 + st.uniform(T * k)).astype(np.float32).reshape(T, k)
        x = fixtures.make_x(seed + T + 10 * k, T, H)
        L.shared = shared_desc if sh else None
        got = _run(L, x, ids, wt)
        ref = oracle_lib.moe_layer(x, ids, wt, experts, shared if sh else None, G2, G1)
        assert L.read_status() == 0, (T, k, sh)
        tol = TOL_BF16 if T * k > 640 else TOL_FP32
        assert _rel_err(got, ref) <= tol, (T, k, sh, _rel_err(got, ref))


def test_tensor_core_path_odd_widths(P, oracle_lib):
    """The tcgen05 path on hidden 768 (three 256-input columns per row tile)
    with experts of widths 256, 512 and 768 in one call (down contractions of
    4, 8 and 12 steps of 64 inputs; 2 to 6 row tiles of 128) and a shared
    expert of width 512: 300 tokens x top-4 = 1200 pairs."""
    H, E, k, T = 768, 12, 4, 300
    seed = 7070
    widths = [256, 512, 768]
    g2, g1 = fixtures.make_grid(seed, 1), fixtures.make_grid(seed, 2)
    experts = [fixtures.make_expert(seed, 1 + (e % 2), H, widths[e % 3], e) for e in range(E)]
    shared = fixtures.make_expert(seed, 2, H, 512, 999)
    L = P.MoeLayer(H, E, 768, T, k, g2, g1, pool_bytes=(E + 2) * fixtures.expert_bytes(1, H, 768) + 4096)
    assert L.upload(list(range(E)), experts) == 0
    assert L.set_shared(shared) == 0
    st = fixtures.Stream(seed, 9)
    ids = np.stack([st.randint(k, E) for _ in range(T)]).astype(np.int32)
    wt = (0.1 + st.uniform(T * k)).astype(np.float32).reshape(T, k)
    x = fixtures.make_x(seed, T, H)
    got = _run(L, x, ids, wt)
    ref = oracle_lib.moe_layer(x, ids, wt, experts, shared, oracle_lib.expand_grid(1, g2),
                               oracle_lib.expand_grid(2, g1))
    assert L.read_status() == 0
    assert _rel_err(got, ref) <= TOL_BF16


@pytest.mark.parametrize("cfg,T", [(2, None), (4, 9), (5, 200)])
def test_host_buffer_entry_point_matches_device_call(P, oracle_lib, cfg, T):
    """redlite_moe_layer_host (packed host inputs -> device, the layer, out ->
    host, on the table's stream) gives redlite_moe_layer's results, twice in a
    row, on the fused decode path (1 and 9 tokens) and on the tensor-core path
    (200 tokens); the first call also matches the fp64 oracle."""
    from bench import pack_inputs

    w = fixtures.workload(cfg, n_tokens=T) if T else fixtures.workload(cfg)
    L = layer_for_workload(w)
    n, H, k = w.x.shape[0], w.hidden, w.top_k
    ref = _run(L, w.x, w.ids, w.weights)
    hin = torch.from_numpy(pack_inputs(w.x, w.ids, w.weights)).pin_memory()
    assert hin.numel() == P.redlite_moe_host_input_bytes(H, n, k)
    din = torch.empty(hin.numel(), dtype=torch.uint8, device="cuda")
    dout = torch.empty((n, H), dtype=torch.float32, device="cuda")
    hout = torch.empty((n, H), dtype=torch.float32).pin_memory()
    tol = 1e-4 if cfg != 5 else 2e-2
    for i in range(2):
        hout.fill_(float("nan"))
        rc = P.redlite_moe_layer_host(hin, din, n, k, L.table, L.shared, dout, hout)
        assert rc == P.REDLITE_OK
        L.stream.synchronize()
        got = hout.numpy().astype(np.float64)
        assert np.isfinite(got).all()
        assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()  # up to the order of fp32 atomic adds
        if i == 0:
            assert _rel_err(got, oracle_lib.workload_layer(w)) <= tol
    assert L.read_status() == 0


@pytest.mark.parametrize("cfg,T", [(2, None), (5, 200)])
def test_two_workspaces_on_two_streams(P, cfg, T):
    """Two tables over the same resident experts, each with its own workspace
    and stream, take calls in turn (host-buffer entry point) and overlap on
    the device: every call gives the single-stream result, on the fused
    decode path and on the tensor-core path."""
    from bench import pack_inputs

    w = fixtures.workload(cfg, n_tokens=T) if T else fixtures.workload(cfg)
    L = layer_for_workload(w)
    n, H, k = w.x.shape[0], w.hidden, w.top_k
    ref = _run(L, w.x, w.ids, w.weights)
    streams = [L.stream, torch.cuda.Stream()]
    t2 = P.redlite_moe_table.from_buffer_copy(bytes(L.table))
    ws2 = torch.zeros(L.workspace.numel(), dtype=torch.uint8, device="cuda")
    t2.workspace, t2.stream = ws2.data_ptr(), streams[1].cuda_stream
    assert P.redlite_moe_workspace_reset(t2) == P.REDLITE_OK
    tables = [L.table, t2]
    packed = pack_inputs(w.x, w.ids, w.weights)
    hin = [torch.from_numpy(packed).pin_memory() for _ in range(2)]
    din = [torch.empty(hin[0].numel(), dtype=torch.uint8, device="cuda") for _ in range(2)]
    dout = [torch.empty((n, H), dtype=torch.float32, device="cuda") for _ in range(2)]
    hout = [[torch.full((n, H), float("nan")).pin_memory() for _ in range(2)] for _ in range(4)]
    torch.cuda.synchronize()
    for i in range(8):
        p = i & 1
        rc = P.redlite_moe_layer_host(hin[p], din[p], n, k, tables[p], L.shared, dout[p], hout[i >> 1][p])
        assert rc == P.REDLITE_OK
    torch.cuda.synchronize()
    for row in hout:
        for h in row:
            got = h.numpy().astype(np.float64)
            assert np.isfinite(got).all()
            assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()
    assert L.read_status() == 0


@pytest.mark.parametrize("cfg", [2, 4])
def test_fused_decode_is_repeatable(P, cfg):
    """100 calls of the fused decode kernel on the same inputs agree up to the
    order of the fp32 atomic additions into out: a stage refilled before all
    its readers were done, an h slice read before it was complete, or a
    stale counter set would show as a large difference in some call."""
    w = fixtures.workload(cfg)
    L = layer_for_workload(w)
    x, ids, wt = _dev(w.x), _dev(w.ids), _dev(w.weights)
    outs = []
    for _ in range(100):
        outs.append(L(x, ids, wt))
    torch.cuda.synchronize()
    assert L.read_status() == 0
    ref = outs[0].cpu().numpy().astype(np.float64)
    scale = np.abs(ref).max()
    for o in outs[1:]:
        assert np.abs(o.cpu().numpy().astype(np.float64) - ref).max() <= 1e-5 * scale


@pytest.mark.parametrize("H,F,T,k,with_shared", [(768, 512, 1, 6, False), (768, 256, 5, 4, True),
                                                 (1280, 512, 1, 8, True), (1280, 256, 3, 6, False),
                                                 (1280, 256, 1, 8, False), (1792, 1280, 1, 3, False)])
def test_fused_decode_odd_block_counts(P, oracle_lib, H, F, T, k, with_shared):
    """The fused decode kernel on hidden sizes whose 256-input block count is
    not a power of two (768: 3 blocks, items of two row tiles with some warps
    idle; 1280: 5 blocks, items of one tile; 1792: 7), tiled widths 256 to
    1280, one and several tokens, with and without a shared expert, against
    the fp64 oracle.  On 148 SMs the last two sit on either side of the
    split's few-down-items rule: 128 gate/up and 40 down items (exactly two
    down items for each of the 20 CTAs without an extra gate/up item), and
    240 and 114 (two more than such CTAs can take in pairs: time slots)."""
    E, seed = 16, 8080 + H + F + T
    g2, g1 = fixtures.make_grid(seed, 1), fixtures.make_grid(seed, 2)
    experts = [fixtures.make_expert(seed, 1 + (e % 2), H, F, e) for e in range(E)]
    shared = fixtures.make_expert(seed, 2, H, F, 999) if with_shared else None
    L = P.MoeLayer(H, E, F, T, k, g2, g1, pool_bytes=(E + 2) * fixtures.expert_bytes(1, H, F) + 4096)
    assert L.upload(list(range(E)), experts) == 0
    if with_shared:
        assert L.set_shared(shared) == 0
    assert L.table.min_ffn >= 256  # the tiled fast path
    st = fixtures.Stream(seed, 3)
    ids = np.stack([np.argsort(st.uniform(E))[:k] for _ in range(T)]).astype(np.int32)
    wt = (0.1 + st.uniform(T * k)).astype(np.float32).reshape(T, k)
    x = fixtures.make_x(seed, T, H)
    got = _run(L, x, ids, wt)
    ref = oracle_lib.moe_layer(x, ids, wt, experts, shared, oracle_lib.expand_grid(1, g2),
                               oracle_lib.expand_grid(2, g1))
    assert L.read_status() == 0
    assert _rel_err(got, ref) <= TOL_FP32
