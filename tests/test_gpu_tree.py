"""Draft-tree attention (mla_decode_attn_tree) against the float64 oracle.

EAGLE-style speculative decoding drafts several tokens as a tree (the
Perplexity write-up's future-work section); each draft attends the
committed prefix, its ancestors and itself.  Random trees of up to 8
drafts, drafts straddling page boundaries, split and unsplit rows; the
chain tree must give the causal result and a star tree one-token decodes.
Tolerance: relative Frobenius <= 5e-3 and max abs <= 2e-2 on `out`."""
import numpy as np
import pytest
import torch

from head_latent_attention_04_b200 import workloads as W
from oracle import mla_oracle as O
from tests.gpu_helpers import check_out, oracle_rows, rel_fro, run_gpu

pytestmark = pytest.mark.gpu


def _run_tree(w, masks, num_clusters):
    from head_latent_attention_04_b200 import mla
    dev = torch.device("cuda")
    wd = w.to(dev)
    bt = torch.as_tensor(w.block_table, dtype=torch.int32, device=dev)
    dec = mla.Decoder(w.seq_lens, w.s_q, w.n_heads, w.max_blocks, w.num_blocks, dev, causal=False,
                      num_clusters=num_clusters)
    dm = torch.as_tensor(np.asarray(masks, dtype=np.int32).reshape(w.B, w.s_q), device=dev)
    res = dec.run(wd.q_nope, wd.q_rope, wd.kv_pool, bt, wd.w_uk, wd.w_uv, draft_masks=dm)
    torch.cuda.synchronize()
    return dec, res


def _random_parents(rng, s_q):
    return [-1] + [int(rng.integers(-1, i)) for i in range(1, s_q)]


@pytest.mark.parametrize("s_q,lens,clusters", [(2, [2, 65, 300], 4), (3, [3, 64, 66, 129], 74),
                                               (5, [5, 130, 1000, 68], 7), (8, [8, 70, 2000, 129], 74),
                                               (8, [64, 4100], 1)])
def test_random_trees_match_oracle(s_q, lens, clusters):
    rng = np.random.default_rng(s_q * 100 + clusters)
    w = W.make_workload(len(lens), s_q, 128, lens, seed=s_q + 40, pool="scattered:1.5")
    masks = [O.tree_masks(_random_parents(rng, s_q)) for _ in lens]
    dec, res = _run_tree(w, masks, clusters)
    assert res.status.item() == 0
    for b in range(w.B):
        ref = oracle_rows(w, b, draft_masks=masks[b])
        rows = slice(b * s_q, (b + 1) * s_q)
        check_out(res.out[rows], ref["out"])
        check_out(res.o_lat[rows], ref["o_lat"])
        np.testing.assert_allclose(res.lse[rows].cpu().numpy(), ref["lse"], rtol=0, atol=2e-2)


@pytest.mark.parametrize("shape", ["chain", "star"])
def test_chain_and_star(shape):
    s_q, lens = 4, [4, 100, 1025]
    w = W.make_workload(len(lens), s_q, 128, lens, seed=77, pool="permuted")
    parents = [-1, 0, 1, 2] if shape == "chain" else [-1, -1, -1, -1]
    masks = [O.tree_masks(parents)] * len(lens)
    dec, res = _run_tree(w, masks, 6)
    assert res.status.item() == 0
    for b in range(w.B):
        ref = oracle_rows(w, b, draft_masks=masks[b])
        check_out(res.out[b * s_q:(b + 1) * s_q], ref["out"])
    if shape == "chain":   # the causal kernel path gives the same attention
        _, causal = run_gpu(w, num_clusters=6)
        assert rel_fro(res.out.float().cpu().numpy(), causal.out.float().cpu().numpy()) < 5e-3


def test_tree_full_size_mtp_shape():
    """B = 128 sequences x 4 drafts in a fixed tree over the mtp2-like length
    mix; rows of two sequences checked on all heads."""
    w = W.preset_workload("mtp2", s_q=4)
    parents = [-1, 0, 0, 1]
    masks = [O.tree_masks(parents)] * w.B
    dec, res = _run_tree(w, masks, None)
    assert res.status.item() == 0
    out = res.out.float().cpu().numpy()
    assert np.all(np.isfinite(out))
    for b in (3, 77):
        if int(w.seq_lens[b]) > 20000:
            continue
        ref = oracle_rows(w, b, draft_masks=masks[b])
        check_out(out[b * 4:(b + 1) * 4], ref["out"])


@pytest.mark.parametrize("s_q,lens,clusters", [(2, [2, 65, 300], 4), (4, [4, 200, 4100], 74)])
def test_non_causal_plan_without_masks(s_q, lens, clusters):
    """dims->causal = 0 on the plain entry point: every query attends all T_b
    keys, the drafts included -- the oracle with every draft visible to every
    query (all mask bits set)."""
    w = W.make_workload(len(lens), s_q, 128, lens, seed=s_q + 90, pool="scattered:1.5")
    dec, res = run_gpu(w, num_clusters=clusters, causal=False)
    assert res.status.item() == 0
    full = [(1 << s_q) - 1] * s_q
    for b in range(w.B):
        ref = oracle_rows(w, b, draft_masks=full)
        rows = slice(b * s_q, (b + 1) * s_q)
        check_out(res.out[rows], ref["out"])
        np.testing.assert_allclose(res.lse[rows].cpu().numpy(), ref["lse"], rtol=0, atol=2e-2)
