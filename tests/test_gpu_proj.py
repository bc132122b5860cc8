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
