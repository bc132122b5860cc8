"""The projection GEMV (Q8_0-style, Q4_K-style) against the fp64 oracle on the
shapes the pages list for the model's dense projections, plus ragged row
counts and several token counts.  fp32 accumulation: max|gpu - oracle| <=
1e-5 * max|oracle|."""
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


# (qtype, rows = outputs, k = inputs): ssm_ba Q8_0 (2048,64); attn_k / attn_v
# Q4_K (2048,512); ssm_out / attn_output Q4_K (4096,2048); ragged extras
CASES = [(3, 64, 2048, 1), (4, 512, 2048, 1), (4, 2048, 4096, 1), (4, 2048, 4096, 8), (3, 37, 512, 3),
         (4, 37, 768, 5), (3, 1000, 256, 2)]


@pytest.mark.parametrize("qtype,rows,k,T", CASES)
def test_proj_gemv_matches_oracle(P, oracle_lib, qtype, rows, k, T):
    m = fixtures.make_proj_matrix(700 + rows, qtype, rows, k)
    assert m.size == P.redlite_proj_matrix_bytes(qtype, rows, k)
    x = fixtures.make_x(701, T, k)
    W = torch.from_numpy(m).cuda()
    xd = torch.from_numpy(x).cuda()
    y = torch.full((T, rows), float("nan"), dtype=torch.float32, device="cuda")
    assert P.redlite_proj_gemv(qtype, W, rows, k, xd, T, y) == P.REDLITE_OK
    torch.cuda.synchronize()
    got = y.cpu().numpy().astype(np.float64)
    ref = oracle_lib.gemv_proj(qtype, m, rows, k, x)
    assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()


@pytest.mark.parametrize("qtype,rows,k,T,offset", [(3, 96, 2048, 2, 2), (3, 33, 512, 1, 6), (4, 40, 11008, 1, 0),
                                                   (4, 9, 11008, 3, 0)])
def test_proj_gemv_fallback_layouts(P, oracle_lib, qtype, rows, k, T, offset):
    """Matrices the streaming kernel does not take: Q8_0-style at a 2-byte
    (not 16-byte) aligned address, and Q4_K-style rows of more than 6 KB (a
    4-row group above the 24 KB stage).  The per-CTA kernel serves them."""
    m = fixtures.make_proj_matrix(900 + rows, qtype, rows, k)
    buf = torch.zeros(m.size + 64, dtype=torch.uint8, device="cuda")
    buf[offset:offset + m.size] = torch.from_numpy(m).cuda()
    W = buf[offset:offset + m.size]
    x = fixtures.make_x(901, T, k)
    xd = torch.from_numpy(x).cuda()
    y = torch.full((T, rows), float("nan"), dtype=torch.float32, device="cuda")
    assert P.redlite_proj_gemv(qtype, W, rows, k, xd, T, y) == P.REDLITE_OK
    torch.cuda.synchronize()
    got = y.cpu().numpy().astype(np.float64)
    ref = oracle_lib.gemv_proj(qtype, m, rows, k, x)
    assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()
