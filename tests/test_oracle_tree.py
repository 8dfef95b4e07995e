"""Pins of the oracle's draft-tree masks (EAGLE-style speculative decoding,
Perplexity write-up, "Будущая работа" / future work: several drafted tokens
arranged as a tree).  Reading: draft i sees the committed prefix, its
ancestors among the drafts and itself.

Pinned by what must hold whatever the implementation:
  * the masks of a chain are the causal masks, so the tree path reproduces
    the (separately pinned) causal oracle;
  * in a star every draft sees only itself, so each row equals a one-token
    decode over prefix + that draft's own cache row;
  * an independent pure-Python brute force with explicit key lists;
  * hand-written masks of a small tree;
  * a planted mistake (a draft also seeing its sibling) fails the brute force.
"""
import math

import numpy as np
import pytest

from oracle import mla_oracle as O
from oracle.brute import brute_decode


def _rand(rng, B, s_q, H, d, R, k, v, lens):
    caches = [rng.standard_normal((T, k + R)) for T in lens]
    return (rng.standard_normal((B * s_q, H, d)), rng.standard_normal((B * s_q, H, R)), caches,
            rng.standard_normal((k, H, d)) / math.sqrt(k), rng.standard_normal((k, H, v)) / math.sqrt(k))


def test_tree_masks_by_hand():
    #        prefix
    #        /    \
    #       0      1
    #      / \      \
    #     2   3      4
    #     |
    #     5
    m = O.tree_masks([-1, -1, 0, 0, 1, 2])
    assert m == [0b000001, 0b000010, 0b000101, 0b001001, 0b010010, 0b100101]
    assert O.tree_masks([-1, 0, 1, 2]) == [0b1, 0b11, 0b111, 0b1111]      # chain = causal
    with pytest.raises(ValueError):
        O.tree_masks([-1, 1])                                               # parent must come first


@pytest.mark.parametrize("s_q,lens", [(2, [2, 9]), (4, [4, 30]), (8, [8, 70])])
def test_chain_tree_equals_causal(s_q, lens):
    rng = np.random.default_rng(s_q)
    args = _rand(rng, len(lens), s_q, 3, 8, 4, 16, 6, lens)
    chain = O.tree_masks([-1] + list(range(s_q - 1)))
    tree = O.mla_decode(*args, s_q, draft_masks=[chain] * len(lens), chunk=5)
    causal = O.mla_decode(*args, s_q, chunk=7)
    for key in ("out", "lse", "o_lat"):
        np.testing.assert_allclose(tree[key], causal[key], rtol=1e-12, atol=1e-13)


def test_star_tree_equals_one_token_decodes():
    s_q, T = 5, 23
    rng = np.random.default_rng(7)
    args = _rand(rng, 1, s_q, 4, 8, 4, 16, 6, [T])
    q_nope, q_rope, (cache,), w_uk, w_uv = args
    star = O.tree_masks([-1] * s_q)
    got = O.mla_decode(*args, s_q, draft_masks=[star])
    prefix = cache[:T - s_q]
    for i in range(s_q):
        own = np.concatenate([prefix, cache[T - s_q + i:T - s_q + i + 1]])
        want = O.mla_decode(q_nope[i:i + 1], q_rope[i:i + 1], [own], w_uk, w_uv, 1)
        np.testing.assert_allclose(got["out"][i], want["out"][0], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(got["lse"][i], want["lse"][0], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("parents,T", [([-1, -1, 0, 0, 1, 2], 9), ([-1, 0, 0, 2], 4), ([-1], 3)])
def test_tree_matches_brute_force(parents, T):
    s_q = len(parents)
    rng = np.random.default_rng(T + s_q)
    H, d, R, k, v = 2, 4, 2, 8, 4
    args = _rand(rng, 2, s_q, H, d, R, k, v, [T, T + 2])
    scale = 1 / math.sqrt(d + R)
    masks = O.tree_masks(parents)
    other = O.tree_masks([-1] * s_q)
    ref = O.mla_decode(*args, s_q, scale=scale, draft_masks=[masks, other], chunk=3)
    visible = []
    for b, Tb in enumerate([T, T + 2]):
        mk = masks if b == 0 else other
        visible.append([list(range(Tb - s_q)) + [Tb - s_q + j for j in range(s_q) if (mk[i] >> j) & 1]
                        for i in range(s_q)])
    out, lse = brute_decode(args[0].tolist(), args[1].tolist(), [c.tolist() for c in args[2]],
                            args[3].tolist(), args[4].tolist(), s_q, scale, visible=visible)
    np.testing.assert_allclose(ref["out"], np.array(out), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(ref["lse"], np.array(lse), rtol=1e-12, atol=1e-13)
    # a planted mistake: draft 3 also sees a draft that is not its ancestor
    if s_q >= 4:
        bad = list(masks)
        bad[3] |= 1 << next(j for j in range(s_q) if not (masks[3] >> j) & 1)
        wrong = O.mla_decode(*args, s_q, scale=scale, draft_masks=[bad, other])
        assert not np.allclose(wrong["out"], np.array(out), rtol=1e-6)
