"""Seeded input generators: shapes, distributions, page layout (CPU only)."""
import math

import numpy as np
import torch

from head_latent_attention_04_b200 import workloads as W
from oracle import mla_oracle as O


def test_presets_shapes_and_pool():
    w = W.preset_workload("tiny")
    assert (w.B, w.s_q, w.n_heads) == (2, 1, 16)
    assert list(w.seq_lens) == [256, 256]
    assert w.block_table.tolist() == [[0, 1, 2, 3], [4, 5, 6, 7]]        # contiguous pool
    assert w.kv_pool.shape == (8, 64, 576) and w.kv_pool.dtype == torch.bfloat16
    assert w.q_nope.shape == (2, 16, 128) and w.q_rope.shape == (2, 16, 64)
    assert w.w_uk.shape == (512, 16, 128) and w.w_uv.shape == (512, 16, 128)


def test_seeded_and_reproducible():
    a = W.preset_workload("tiny")
    b = W.preset_workload("tiny")
    assert torch.equal(a.kv_pool, b.kv_pool) and torch.equal(a.q_nope, b.q_nope)
    c = W.preset_workload("tiny", seed=99)
    assert not torch.equal(a.kv_pool, c.kv_pool)


def test_value_distributions():
    w = W.make_workload(4, 1, 32, [700, 64, 1, 2000], seed=3, pool="scattered:1.5")
    rows = torch.cat([w.cache_rows(b) for b in range(4)]).float()
    assert abs(rows.mean().item()) < 0.01 and abs(rows.std().item() - 1) < 0.01
    assert abs(w.w_uk.float().std().item() - 1 / math.sqrt(512)) < 2e-3
    assert abs(w.w_uv.float().std().item() - 1 / math.sqrt(512)) < 2e-3
    assert abs(w.q_nope.float().std().item() - 1) < 0.02


def test_page_table_gather_independent():
    """Rebuild each sequence from the pool with explicit per-page copies."""
    w = W.make_workload(3, 2, 4, [130, 64, 5], seed=4, pool="scattered:2")
    assert w.num_blocks == 2 * (3 + 1 + 1)
    used = set()
    for b in range(3):
        T = int(w.seq_lens[b])
        n_pages = -(-T // 64)
        assert np.all(w.block_table[b, n_pages:] == -1)
        pieces = []
        for p in range(n_pages):
            blk = int(w.block_table[b, p])
            assert 0 <= blk < w.num_blocks and blk not in used
            used.add(blk)
            pieces.append(w.kv_pool[blk])
        seq = torch.cat(pieces)
        assert torch.equal(seq[:T], w.cache_rows(b))
        assert torch.all(seq[T:].float() == W.POISON)       # tail of the last page
    for blk in set(range(w.num_blocks)) - used:
        assert torch.all(w.kv_pool[blk].float() == W.POISON)


def test_permutation_invariance_of_oracle_inputs():
    """Same seed, different pool layout: identical cache rows, identical oracle output."""
    a = W.make_workload(2, 1, 4, [100, 70], seed=5, pool="contiguous")
    b = W.make_workload(2, 1, 4, [100, 70], seed=5, pool="scattered:3")
    assert not np.array_equal(a.block_table, b.block_table)
    outs = []
    for w in (a, b):
        caches = [w.cache_rows(i).double().numpy() for i in range(2)]
        assert torch.equal(w.cache_rows(0), a.cache_rows(0))
        outs.append(O.mla_decode(w.q_nope.double().numpy(), w.q_rope.double().numpy(), caches,
                                 w.w_uk.double().numpy(), w.w_uv.double().numpy(), 1,
                                 with_intermediates=False)["out"])
    np.testing.assert_array_equal(outs[0], outs[1])


def test_lognormal_lengths_in_range():
    rng = np.random.default_rng(0)
    T = W.draw_seq_lens("lognormal:4096:1.0:32768", 5000, 2, rng)
    assert T.min() >= 2 and T.max() <= 32768
    assert 3500 < np.median(T) < 4700
