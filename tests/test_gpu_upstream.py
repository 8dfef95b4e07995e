"""Upstream fusions against the float64 oracle: the fused qkv_a_proj (both
down-projections in one launch) and the query up-projection feeding the
first absorption in one kernel (q_nope stays on chip, rounded to bf16 there
as the bf16 path rounds every intermediate).  Tolerance: relative Frobenius
<= 5e-3 and max abs <= 2e-2."""
import math

import numpy as np
import pytest
import torch

from oracle import mla_oracle as O
from tests.gpu_helpers import check_out

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mla():
    from head_latent_attention_04_b200 import mla as m
    return m


def _bf16(shape, std, gen):
    return (torch.randn(shape, generator=gen) * std).to(torch.bfloat16)


@pytest.mark.parametrize("N,H", [(1, 1), (7, 16), (32, 128), (100, 128), (128, 5), (200, 128), (300, 3)])
def test_q_up_absorb_matches_oracle(mla, N, H):
    g = torch.Generator().manual_seed(N * 131 + H)
    c_q = _bf16((N, 1536), 1.0, g)
    w_uq = _bf16((1536, H, 192), 1 / math.sqrt(1536), g)
    w_uk = _bf16((512, H, 128), 1 / math.sqrt(512), g)
    q_lat, q_rope = mla.q_up_absorb(c_q.cuda(), w_uq.cuda(), w_uk.cuda())
    torch.cuda.synchronize()
    qn, qr = O.query_up(c_q.double().numpy(), w_uq.double().numpy())
    want = O.contract(None, "absorb_q", "nhd,khd->nhk", qn, w_uk.double().numpy())
    check_out(q_rope, qr)
    check_out(q_lat, want)


@pytest.mark.parametrize("N", [1, 32, 128, 130, 256, 257, 600])
def test_qkv_a_proj_matches_oracle(mla, N):
    g = torch.Generator().manual_seed(N + 7)
    x = _bf16((N, 7168), 1.0, g)
    w_dq = _bf16((7168, 1536), 1 / math.sqrt(7168), g)
    w_dkv = _bf16((7168, 576), 1 / math.sqrt(7168), g)
    w = torch.cat([w_dq, w_dkv], dim=1).t().contiguous()        # [2112][7168]
    c_q, kv_a = mla.qkv_a_proj(x.cuda(), w.cuda())
    torch.cuda.synchronize()
    want_q, want_kv = O.qkv_down(x.double().numpy(), w_dq.double().numpy(), w_dkv.double().numpy())
    check_out(c_q, want_q)
    check_out(kv_a, want_kv)
