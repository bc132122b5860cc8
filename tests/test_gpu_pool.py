"""The slot pool end to end on the GPU: acquire() makes each selection
resident (H2D fills on a copy stream, slot-table updates), the layer call
that follows on the compute stream sees the filled slots, and the results
match the fp64 oracle.  Checks the cold top-10 counters the pages expect
(10 loads, 30 matrix reads), hits on reuse, LRU eviction with the evicted
experts' slot-table entries cleared (a stale id is reported, not read), and
in-flight protection released by a CUDA event."""
import ctypes

import numpy as np
import pytest
import torch

import fixtures

pytestmark = pytest.mark.gpu

TOL = 1e-4


@pytest.fixture(scope="module")
def P():
    from routed_expert_ffn_iq2_b200 import build

    build.build()
    import routed_expert_ffn_iq2_b200 as P

    return P


def test_pool_feeds_the_layer(P, oracle_lib):
    w = fixtures.workload(2)  # hidden 2048, 512 IQ2_XS-style experts of width 512, top-10
    H, E, F, k = w.hidden, w.n_experts, w.ffn, w.top_k
    sets = fixtures.decode_id_sets(fixtures.SEED_BASE + 2, 4, k, E)
    A, B, C = [list(map(int, s)) for s in sets[:3]]
    cap = 24
    L = P.MoeLayer(H, E, F, 1, k, w.grid_iq2, w.grid_iq1, pool_bytes=16)
    L.table.min_ffn = F
    gb = fixtures.matrix_bytes(1, F, H)
    slot_bytes = 2 * ((gb + 15) // 16 * 16) + fixtures.matrix_bytes(1, H, F)
    slots = torch.zeros(cap * slot_bytes, dtype=torch.uint8, device="cuda")
    host = (P.redlite_moe_expert * E)()
    keep = []
    for e in set(A + B + C):
        ex = w.expert(e)
        mats = [np.ascontiguousarray(P.redlite_moe_pack_matrix(1, r, c, m))
                for m, (r, c) in zip((ex.gate, ex.up, ex.down), ((F, H), (F, H), (H, F)))]
        keep += mats
        host[e] = P.redlite_moe_expert(1, F, *[m.ctypes.data for m in mats])
    pool = P.SlotPool(E, cap)
    copy_s, comp_s = torch.cuda.Stream(), torch.cuda.current_stream()
    g2 = oracle_lib.expand_grid(1, w.grid_iq2)
    x = torch.from_numpy(w.x).cuda()
    wt = torch.from_numpy(w.weights).cuda()

    def run(sel):
        ids = torch.tensor([sel], dtype=torch.int32, device="cuda")
        out = L(x, ids, wt)
        torch.cuda.synchronize()
        return out.cpu().numpy().astype(np.float64)

    def ref(sel):
        experts = [None] * E
        for e in sel:
            experts[e] = w.expert(e)
        return oracle_lib.moe_layer(w.x, np.array([sel], np.int32), w.weights, experts, None, g2, None)

    def acquire(sel):
        rc, tok = pool.acquire(sel, host, H, slots, slot_bytes, L.table_dev, copy_s, comp_s)
        assert rc == P.REDLITE_OK
        return tok

    # cold top-10: 10 loads, 30 matrix copies, then the layer matches the oracle
    tA = acquire(A)
    assert (pool.counters.loads, pool.counters.copies, pool.counters.hits) == (10, 30, 0)
    assert pool.counters.bytes == 10 * fixtures.expert_bytes(1, H, F)
    got = run(A)
    assert L.read_status() == 0
    assert np.abs(got - ref(A)).max() <= TOL * np.abs(ref(A)).max()
    # while A is in flight (not released) its slots cannot be taken: B fits the free 14 slots
    tB = acquire(B)
    assert pool.counters.loads == 20
    assert all(pool.pins(pool.slot_of(e)) == 1 for e in A)
    # C needs 10 slots: 4 free, 6 must be evicted, but A and B are still pinned
    rc, _ = pool.acquire(C, host, H, slots, slot_bytes, L.table_dev, copy_s, comp_s)
    assert rc == P.REDLITE_EAGAIN and pool.counters.loads == 20
    # release both after the work so far (a CUDA event); C then evicts A's least recent experts
    assert pool.release(tA, comp_s) == 0 and pool.release(tB, comp_s) == 0
    torch.cuda.synchronize()
    tC = acquire(C)
    assert pool.counters.loads == 30 and pool.counters.evictions == 6
    evicted = [e for e in A if pool.slot_of(e) < 0]
    assert len(evicted) == 6 and all(pool.slot_of(e) >= 0 for e in B + C)
    got = run(C)
    assert L.read_status() == 0
    assert np.abs(got - ref(C)).max() <= TOL * np.abs(ref(C)).max()
    # a stale selection (A without acquiring): the evicted experts are reported, not read
    run(A)
    assert L.read_status() & P.REDLITE_STATUS_BAD_EXPERT
    L.clear_status()
    pool.release(tC, comp_s)
    torch.cuda.synchronize()
    # A again: 4 hits, 6 loads, and the layer matches the oracle
    hits0, loads0 = pool.counters.hits, pool.counters.loads
    acquire(A)
    assert pool.counters.hits - hits0 == 4 and pool.counters.loads - loads0 == 6
    got = run(A)
    assert L.read_status() == 0
    assert np.abs(got - ref(A)).max() <= TOL * np.abs(ref(A)).max()
    pool.close()
    del keep


def test_pool_pipelined_calls_with_evictions(P, oracle_lib):
    """Sixteen top-10 calls over 40 experts through a 24-slot pool, enqueued
    back to back: each call's slots are released by an event recorded after
    it, with no host synchronisation in between except when the pool reports
    every candidate slot in flight (EAGAIN).  A fill for a later selection
    must never land in a slot that an earlier, still running call reads, so
    every call's output matches the fp64 oracle at the end."""
    w = fixtures.workload(2)
    H, E, F, k = w.hidden, w.n_experts, w.ffn, w.top_k
    st = fixtures.Stream(fixtures.SEED_BASE + 2, 77)
    sels = [[12 * u + 3 for u in fixtures.draw_distinct_nonadjacent(st, k, 40)] for _ in range(16)]
    cap = 24
    L = P.MoeLayer(H, E, F, 1, k, w.grid_iq2, w.grid_iq1, pool_bytes=16)
    L.table.min_ffn = F
    gb = fixtures.matrix_bytes(1, F, H)
    slot_bytes = 2 * ((gb + 15) // 16 * 16) + fixtures.matrix_bytes(1, H, F)
    slots = torch.zeros(cap * slot_bytes, dtype=torch.uint8, device="cuda")
    host = (P.redlite_moe_expert * E)()
    keep = []
    for e in sorted(set(sum(sels, []))):
        ex = w.expert(e)
        mats = [np.ascontiguousarray(P.redlite_moe_pack_matrix(1, r, c, m))
                for m, (r, c) in zip((ex.gate, ex.up, ex.down), ((F, H), (F, H), (H, F)))]
        keep += mats
        host[e] = P.redlite_moe_expert(1, F, *[m.ctypes.data for m in mats])
    pool = P.SlotPool(E, cap)
    copy_s, comp_s = torch.cuda.Stream(), torch.cuda.current_stream()
    x = torch.from_numpy(w.x).cuda()
    wt = torch.from_numpy(w.weights).cuda()
    outs, waits = [], 0
    for sel in sels:
        ids = torch.tensor([sel], dtype=torch.int32, device="cuda")
        while True:
            rc, tok = pool.acquire(sel, host, H, slots, slot_bytes, L.table_dev, copy_s, comp_s)
            if rc == P.REDLITE_OK:
                break
            assert rc == P.REDLITE_EAGAIN
            waits += 1
            assert waits < 64
            comp_s.synchronize()  # the calls in flight end; their events complete
        outs.append(L(x, ids, wt))
        assert pool.release(tok, comp_s) == 0
    torch.cuda.synchronize()
    assert L.read_status() == 0
    assert pool.counters.evictions > 0 and pool.counters.hits > 0
    g2 = oracle_lib.expand_grid(1, w.grid_iq2)
    for sel, o in zip(sels, outs):
        experts = [None] * E
        for e in sel:
            experts[e] = w.expert(e)
        ref = oracle_lib.moe_layer(w.x, np.array([sel], np.int32), w.weights, experts, None, g2, None)
        got = o.cpu().numpy().astype(np.float64)
        assert np.abs(got - ref).max() <= TOL * np.abs(ref).max()
    pool.close()
    del keep
