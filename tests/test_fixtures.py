"""Sanity of the seeded input recipe (not of the method)."""
import numpy as np

import fixtures


def test_streams_deterministic_and_distinct():
    a = fixtures.Stream(1, 2, 3).u64(16)
    b = fixtures.Stream(1, 2, 3).u64(16)
    c = fixtures.Stream(1, 2, 4).u64(16)
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    s = fixtures.Stream(1, 2, 3)
    assert np.array_equal(np.concatenate([s.u64(5), s.u64(11)]), a)


def test_normal_moments():
    z = fixtures.Stream(7, 1).normal(200000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01


def test_decode_routing_recipe():
    for cfg in (2, 3):
        w = fixtures.workload(cfg)
        ids = w.ids[0].tolist()
        assert len(set(ids)) == 10
        assert all(abs(a - b) != 1 for a in ids for b in ids)
        assert np.all(w.weights > 0) and abs(float(w.weights.sum()) - 1) < 1e-6


def test_batched_routing_recipe():
    w = fixtures.workload(4)
    assert w.ids.shape == (64, 10)
    for t in range(64):
        assert len(set(w.ids[t].tolist())) == 10
    np.testing.assert_allclose(w.weights.sum(1), 1, rtol=1e-6)
    assert np.all(np.diff(w.weights, axis=1) <= 0)  # top-k in descending probability
    assert set(np.unique(w.qtypes[w.ids]).tolist()) == {1, 2}


def test_prefill_routing_skewed():
    w = fixtures.workload(5, n_tokens=4096)
    cnt = np.bincount(w.ids.reshape(-1), minlength=512)
    assert cnt.sum() == 40960 and cnt.max() > 2000 and (cnt < 16).sum() > 50
    for t in range(0, 4096, 97):
        assert len(set(w.ids[t].tolist())) == 10


def test_disjoint_id_sets():
    s = fixtures.decode_id_sets(fixtures.SEED_BASE + 2, 48, 10, 512)
    assert len(set(s.reshape(-1).tolist())) == 480


def test_block_scale_ranges():
    for q, lo, hi in ((1, 2.0 ** -12, 2.0 ** -10), (2, 2.0 ** -9, 2.0 ** -7)):
        m = fixtures.make_matrix(3, q, 512, 2048, 0).reshape(-1, fixtures.BLOCK_BYTES[q])
        d = (m[:, 0].astype(np.uint16) | (m[:, 1].astype(np.uint16) << 8)).view(np.float16).astype(np.float64)
        assert d.min() >= lo and d.max() < hi
