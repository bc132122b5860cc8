"""The allocation-free entry point (redlite_moe_layer_noalloc) gives the same
results as redlite_moe_layer, called through the C ABI twice in a row.

Some callers cannot allocate device memory for a workspace (for example a
plugin inside a host application that owns the whole device-memory budget);
this entry point keeps the kernel's scratch in an array the library holds.
The file is named to be collected last."""
import numpy as np
import pytest
import torch

import fixtures
from bench import layer_for_workload

pytestmark = pytest.mark.gpu

TOL = 1e-4  # same bound as the fp32-accumulate layer tests


@pytest.fixture(scope="module")
def P():
    from routed_expert_ffn_iq2_b200 import build

    build.build()
    import routed_expert_ffn_iq2_b200 as P

    return P


@pytest.mark.parametrize("cfg,T", [(2, None), (4, 9)])
def test_no_alloc_matches_workspace_entry_point(P, cfg, T):
    w = fixtures.workload(cfg, n_tokens=T) if T else fixtures.workload(cfg)
    L = layer_for_workload(w)
    x = torch.from_numpy(w.x).cuda()
    ids = torch.from_numpy(w.ids).cuda()
    wt = torch.from_numpy(w.weights).cuda()
    ref = L(x, ids, wt)
    torch.cuda.synchronize()
    ref = ref.cpu().numpy().astype(np.float64)
    for _ in range(2):
        out = torch.full_like(x[:, :w.hidden], float("nan"))
        rc = P.redlite_moe_layer_noalloc(x, x.shape[0], ids, wt, w.top_k, L.table, L.shared, out)
        torch.cuda.synchronize()
        assert rc == P.REDLITE_OK
        got = out.cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all()
        assert np.abs(got - ref).max() <= TOL * np.abs(ref).max()
    assert L.read_status() == 0


def test_no_alloc_rejects_what_it_cannot_take(P):
    w = fixtures.workload(1)  # expert width 64: not a fused-kernel shape
    L = layer_for_workload(w)
    x = torch.from_numpy(w.x).cuda()
    ids = torch.from_numpy(w.ids).cuda()
    wt = torch.from_numpy(w.weights).cuda()
    out = torch.empty_like(x)
    rc = P.redlite_moe_layer_noalloc(x, 1, ids, wt, w.top_k, L.table, None, out)
    assert rc == P.REDLITE_EUNSUPPORTED


def test_no_alloc_refusals_leave_out_untouched(P):
    """Calls the fixed scratch array cannot serve, and malformed shared
    experts, are refused on the host before anything is enqueued: out keeps
    its contents and the status word stays clear."""
    w = fixtures.workload(4)  # 64 tokens x top-10 + shared expert
    L = layer_for_workload(w)
    x = torch.from_numpy(w.x).cuda()
    ids = torch.from_numpy(w.ids).cuda()
    wt = torch.from_numpy(w.weights).cuda()
    out = torch.full_like(x, 3.5)
    # declared max_ffn 2048: 704 pairs x 2048 fp32 h values do not fit 4 MiB
    big = P.redlite_moe_table.from_buffer_copy(bytes(L.table))
    big.max_ffn = 2048
    rc = P.redlite_moe_layer_noalloc(x, x.shape[0], ids, wt, w.top_k, big, L.shared, out)
    assert rc == P.REDLITE_ENOMEM
    bad = P.redlite_moe_expert(L.shared.qtype, L.shared.ffn, L.shared.gate + 8, L.shared.up, L.shared.down)
    rc = P.redlite_moe_layer_noalloc(x, x.shape[0], ids, wt, w.top_k, L.table, bad, out)
    assert rc == P.REDLITE_EINVAL
    bad = P.redlite_moe_expert(7, L.shared.ffn, L.shared.gate, L.shared.up, L.shared.down)
    rc = P.redlite_moe_layer_noalloc(x, x.shape[0], ids, wt, w.top_k, L.table, bad, out)
    assert rc == P.REDLITE_EINVAL
    torch.cuda.synchronize()
    assert bool((out == 3.5).all())
    assert L.read_status() == 0
