"""Pins of the oracle's upstream steps: the query up-projection from c^Q
(W^UQ, notes section 2.1, with the RoPE query columns q_b_proj also yields)
and the fused down-projection qkv_a_proj (Perplexity write-up, "MLA layer":
q_a_proj and kv_a_proj merged into one product).

Checked against: scalar brute force on tiny shapes, the first absorption's
own W^UQ path (orders 1, 2 and 3 of the logits agree when q_nope comes from
query_up), the FLOP term 2bshdq of the notes, and a planted transpose."""
import math

import numpy as np
import pytest

from oracle import mla_oracle as O


def _brute_q(c_q, W):
    n, qd = len(c_q), len(c_q[0])
    h, f = len(W[0]), len(W[0][0])
    out = [[[0.0] * f for _ in range(h)] for _ in range(n)]
    for a in range(n):
        for b in range(h):
            for c in range(f):
                acc = 0.0
                for j in range(qd):
                    acc += c_q[a][j] * W[j][b][c]
                out[a][b][c] = acc
    return np.array(out)


def test_query_up_matches_brute_force():
    rng = np.random.default_rng(1)
    c_q = rng.standard_normal((3, 5))
    W = rng.standard_normal((5, 2, 6))              # d_nope = 4, R = 2
    qn, qr = O.query_up(c_q, W, d_nope=4)
    full = _brute_q(c_q.tolist(), W.tolist())
    np.testing.assert_allclose(qn, full[:, :, :4], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(qr, full[:, :, 4:], rtol=1e-13, atol=1e-13)
    bad, _ = O.query_up(c_q, W.transpose(0, 1, 2)[:, ::-1, :].copy(), d_nope=4)   # heads swapped
    assert not np.allclose(bad, full[:, :, :4])


def test_query_up_feeds_the_first_absorption():
    """Logits from (query_up -> order 2) equal the first absorption's own
    W^UQ path in orders 1, 2 and 3."""
    rng = np.random.default_rng(2)
    b, s, t, q, h, d, k = 1, 3, 7, 12, 3, 4, 8
    c_q = rng.standard_normal((b * s, q))
    W_UQ = rng.standard_normal((q, h, d + 2)) / math.sqrt(q)
    W_UK = rng.standard_normal((k, h, d)) / math.sqrt(k)
    ckv = rng.standard_normal((b, t, k))
    qn, _ = O.query_up(c_q, W_UQ, d_nope=d)
    via_query = O.first_absorption_logits(2, qn.reshape(b, s, h, d), W_UK, ckv)
    for order in (1, 2, 3):
        ref = O.first_absorption_logits(order, c_q.reshape(b, s, q), W_UK, ckv, W_UQ=W_UQ[:, :, :d])
        np.testing.assert_allclose(via_query, ref, rtol=1e-12, atol=1e-12)


def test_query_up_flops_are_the_2bshdq_term():
    c = O.FlopCounter(dry=True)
    O.query_up(O.Shape((32, 1536)), O.Shape((1536, 128, 128)), d_nope=128, counter=c)
    assert c.terms["uq"] == 2 * 32 * 128 * 128 * 1536       # notes: 2bshdq with b*s = 32
    c = O.FlopCounter(dry=True)
    qn, qr = O.query_up(O.Shape((32, 1536)), O.Shape((1536, 128, 192)), d_nope=128, counter=c)
    assert qn.shape == (32, 128, 128) and qr.shape == (32, 128, 64)


def test_qkv_down_is_both_down_projections():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 9))
    W_DQ = rng.standard_normal((9, 5))
    W_DKV = rng.standard_normal((9, 7))
    c_q, kv = O.qkv_down(x, W_DQ, W_DKV)
    for a in range(4):
        for j in range(5):
            assert abs(c_q[a, j] - sum(x[a, e] * W_DQ[e, j] for e in range(9))) < 1e-12
        for j in range(7):
            assert abs(kv[a, j] - sum(x[a, e] * W_DKV[e, j] for e in range(9))) < 1e-12
    # one product over the concatenated weight gives the same rows
    both = x @ np.concatenate([W_DQ, W_DKV], axis=1)
    np.testing.assert_allclose(both[:, :5], c_q, rtol=1e-13)
    np.testing.assert_allclose(both[:, 5:], kv, rtol=1e-13)
