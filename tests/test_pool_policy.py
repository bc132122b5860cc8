"""The slot pool's policy, host only (no GPU): the plain model in
oracle/lru.py pinned to hand-worked sequences (tests/golden/
pool_sequences.json) and to invariants; the library's pool compared with the
model decision by decision on hand-worked and random sequences."""
import json
import os

import numpy as np
import pytest

import fixtures
from oracle.lru import EAGAIN, ENOMEM, OK, LruModel

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "pool_sequences.json")


@pytest.fixture(scope="module")
def P():
    from routed_expert_ffn_iq2_b200 import build

    build.build()
    import routed_expert_ffn_iq2_b200 as P

    return P


def _play(pool, case):
    tokens = []
    for st in case["steps"]:
        if "complete" in st:
            assert pool.complete(tokens[st["complete"] - 1]) == OK
            continue
        rc, slots, ev, miss, tok = pool.plan(st["ids"])
        if "error" in st:
            assert rc == st["error"], (case["name"], st)
            tokens.append(None)
            continue
        assert rc == OK, (case["name"], st, rc)
        assert list(slots) == st["slots"], (case["name"], st, slots)
        assert [bool(m) for m in miss] == st["miss"], (case["name"], st, miss)
        assert list(ev) == st["evicted"], (case["name"], st, ev)
        tokens.append(tok)


def test_model_golden_sequences():
    for case in json.load(open(GOLDEN))["cases"]:
        _play(LruModel(case["n_experts"], case["capacity"]), case)


def test_library_golden_sequences(P):
    for case in json.load(open(GOLDEN))["cases"]:
        pool = P.SlotPool(case["n_experts"], case["capacity"])
        _play(pool, case)
        pool.close()


def test_model_invariants():
    """Random traffic: residency is a bijection within capacity, a selection is
    resident after its plan, and a pinned slot never changes its expert."""
    st = fixtures.Stream(99, 1)
    m = LruModel(64, 12)
    held = []
    for step in range(600):
        k = 1 + int(st.randint(1, 10)[0])
        ids = [int(v) for v in st.randint(k, 64)]
        before = {s: m.slot_expert[s] for s in range(12) if m.pins[s] > 0}
        rc, slots, ev, miss, tok = m.plan(ids)
        if rc == OK:
            assert all(m.expert_slot[e] == s for e, s in zip(ids, slots))
            held.append(tok)
        else:
            assert rc in (EAGAIN, ENOMEM)
        for s, e in before.items():
            assert m.slot_expert[s] == e
        assert len(m.expert_slot) <= 12
        assert sorted(m.expert_slot.values()) == sorted(s for s in range(12) if m.slot_expert[s] >= 0)
        if held and st.uniform(1)[0] < 0.6:
            m.complete(held.pop(int(st.randint(1, len(held))[0])))


@pytest.mark.parametrize("seed,E,cap", [(1, 32, 8), (2, 512, 40), (3, 16, 16), (4, 100, 10)])
def test_library_matches_model_on_random_traffic(P, seed, E, cap):
    st = fixtures.Stream(seed, 7)
    m, pool = LruModel(E, cap), P.SlotPool(E, cap)
    mt, pt = [], []
    for step in range(400):
        k = 1 + int(st.randint(1, min(cap + 2, 12))[0])
        ids = [int(v) for v in st.randint(k, E)]
        want = m.plan(ids)
        got = pool.plan(ids)
        assert got[0] == want[0], (step, ids)
        if want[0] == OK:
            assert got[1:4] == want[1:4], (step, ids)
            mt.append(want[4])
            pt.append(got[4])
        if mt and st.uniform(1)[0] < 0.5:
            j = int(st.randint(1, len(mt))[0])
            assert m.complete(mt.pop(j)) == OK and pool.complete(pt.pop(j)) == OK
        for s in range(cap):
            assert pool.pins(s) == m.pins[s]
    for e in range(E):
        assert pool.slot_of(e) == m.expert_slot.get(e, -1)
    pool.close()


def test_library_rejects(P):
    pool = P.SlotPool(8, 2)
    assert pool.plan([8])[0] == -1 and pool.plan([-1])[0] == -1
    assert pool.complete(12345) == -1
    pool.close()
