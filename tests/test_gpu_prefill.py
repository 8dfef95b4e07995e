"""Prefill and chunked prefill in order 1 (mla_prefill_up_proj +
mla_prefill_attn) against the float64 oracle.

The oracle is the same un-absorbed decode oracle with s query tokens: the
last s of T cached tokens attend causally ("MLA Matrix Absorption
Analysis" section 2.4.1: order 1 is the cheaper order when t = s).
Tolerance: relative Frobenius <= 5e-3 and max abs <= 2e-2 on out, K and V."""
import numpy as np
import pytest
import torch

from head_latent_attention_04_b200 import workloads as W
from oracle import mla_oracle as O
from tests.gpu_helpers import check_out

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mla():
    from head_latent_attention_04_b200 import mla as m
    return m


def _setup(T, s, H, seed, poison=W.POISON):
    w = W.make_workload(1, s, H, [T], seed=seed, pool="scattered:1.5", poison=poison)
    dev = torch.device("cuda")
    wd = w.to(dev)
    row = torch.as_tensor(w.block_table[0], dtype=torch.int32, device=dev).contiguous()
    return w, wd, row


@pytest.mark.parametrize("T,H", [(1, 16), (63, 128), (64, 7), (65, 128), (300, 128), (1000, 32)])
def test_up_projection_matches_oracle(mla, T, H):
    w, wd, row = _setup(T, 1, H, seed=T + H)
    k, v = mla.prefill_up_proj(wd.kv_pool, row, T, wd.w_uk, wd.w_uv)
    torch.cuda.synchronize()
    ckv = w.cache_rows(0)[:, :512].double().numpy()
    want_k = O.contract(None, "uk", "tk,khd->thd", ckv, w.w_uk.double().numpy())
    want_v = O.contract(None, "uv", "tk,khv->thv", ckv, w.w_uv.double().numpy())
    check_out(k, want_k)
    check_out(v, want_v)


def _check_prefill(mla, T, s, H, seed, heads=None, poison=W.POISON):
    w, wd, row = _setup(T, s, H, seed, poison)
    lse = torch.empty((s, H), dtype=torch.float32, device="cuda")
    out = mla.prefill(wd.q_nope, wd.q_rope, wd.kv_pool, row, T, wd.w_uk, wd.w_uv, lse=lse)
    torch.cuda.synchronize()
    ref = O.mla_decode(w.q_nope.double().numpy(), w.q_rope.double().numpy(), [w.cache_rows(0).double().numpy()],
                       w.w_uk.double().numpy(), w.w_uv.double().numpy(), s, heads=heads, with_intermediates=False)
    got = out if heads is None else out[:, heads]
    check_out(got, ref["out"])
    got_l = lse.cpu().numpy() if heads is None else lse[:, heads].cpu().numpy()
    np.testing.assert_allclose(got_l, ref["lse"], rtol=0, atol=2e-2)


@pytest.mark.parametrize("T,H", [(1, 16), (2, 128), (64, 128), (127, 16), (128, 128), (129, 128), (300, 64)])
def test_full_prefill_matches_oracle(mla, T, H):
    _check_prefill(mla, T, T, H, seed=T * 3 + H)


@pytest.mark.parametrize("T,s", [(1000, 1), (1000, 128), (1000, 300), (4097, 129)])
def test_chunked_prefill_matches_oracle(mla, T, s):
    """A chunk of s tokens after a prefix of T - s: every chunk query sees the
    whole prefix and the chunk causally."""
    _check_prefill(mla, T, s, 128, seed=T + s)


@pytest.mark.parametrize("poison", [float("nan"), float("inf")])
def test_prefill_ignores_non_finite_page_tails(mla, poison):
    _check_prefill(mla, 130, 130, 32, seed=5, poison=poison)
    _check_prefill(mla, 200, 70, 32, seed=6, poison=poison)


def test_full_size_prefill_4k_sampled_heads(mla):
    """A 4096-token prefill with 128 heads (32 query tiles x 128 heads),
    checked on heads from every lane quarter of the up-projection tiles."""
    _check_prefill(mla, 4096, 4096, 128, seed=11, heads=[0, 45, 90, 127])
