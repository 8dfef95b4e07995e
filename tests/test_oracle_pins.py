"""Pins of the float64 oracle against what the pages and mathematics fix (CPU only).

Each test ties the oracle to something other than itself: integers the pages
print (tests/golden/flop_pins.json), closed forms, library routines, an
independent pure-Python brute force, and algebraic identities between the
notes' evaluation orders.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special

from oracle import mla_oracle as O
from oracle.brute import brute_decode

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "flop_pins.json")))
DIMS = GOLD["dims"]
FIRST = {1: ("uq", "uk", "qk"), 2: ("uq", "absorb_q", "qk_lat"), 3: ("pre_uq_uk", "cq_pre", "qk_lat")}
SECOND = {1: ("uv", "pv", "o"), 2: ("pv_lat", "out_uv", "o"), 3: ("pre_o_uv", "pv_lat", "o_pre")}


def _flops(order, b, s, t, which, **kw):
    c = O.step_flops(order, b, s, t, h=DIMS["h"], d=DIMS["d"], k=DIMS["k"], v=DIMS["v"],
                     q=DIMS["q"], e=DIMS["e"] if order == 3 or kw.get("with_o") else None)
    labels = FIRST[order] if which == "first" else SECOND[order]
    return c.total(*labels)


# ---------------------------------------------------------------- FLOP pins
@pytest.mark.parametrize("s", [1, 2, 7, 64, 1000])
def test_first_order1_vs_order2_prefill_printed(s):
    g = GOLD["first_order1_minus_order2_prefill"]
    assert _flops(1, 1, s, s, "first") - _flops(2, 1, s, s, "first") == g["coef_s2"] * s * s


@pytest.mark.parametrize("t", [1, 2, 100, 4096, 5000, 131072])
def test_first_order1_vs_order2_decode_printed(t):
    g = GOLD["first_order1_minus_order2_decode"]
    diff = _flops(1, 1, 1, t, "first") - _flops(2, 1, 1, t, "first")
    assert diff == g["a"] * (t - 1) + g["c"] * t
    assert diff == g["slope"] * t + g["intercept"]


@pytest.mark.parametrize("b,s,t", [(1, 1, 1), (1, 1, 4096), (3, 2, 50), (32, 1, 4096)])
def test_first_order2_vs_order3_printed(b, s, t):
    g = GOLD["first_order2_minus_order3"]
    diff = _flops(2, b, s, t, "first") - _flops(3, b, s, t, "first")
    assert diff == g["slope_bs"] * b * s + g["intercept"]


def test_pre_absorbed_weight_size_printed():
    g = GOLD["first_order2_minus_order3"]
    W = O.contract(O.FlopCounter(dry=True), "pre_uq_uk", "qhd,khd->hqk",
                   O.Shape((DIMS["q"], DIMS["h"], DIMS["d"])), O.Shape((DIMS["k"], DIMS["h"], DIMS["d"])))
    assert math.prod(W.shape) == g["pre_absorbed_elements"]
    assert DIMS["q"] * DIMS["h"] * DIMS["d"] + DIMS["k"] * DIMS["h"] * DIMS["d"] == g["factored_elements"]


@pytest.mark.parametrize("b,s,t", [(1, 1, 1), (1, 1, 5000), (1, 9, 9), (2, 2, 300)])
def test_second_order1_vs_order2_matches_first(b, s, t):
    d2 = _flops(1, b, s, t, "second") - _flops(2, b, s, t, "second")
    d1 = _flops(1, b, s, t, "first") - _flops(2, b, s, t, "first")
    assert GOLD["second_order1_minus_order2"]["same_as"] == "first_order1_minus_order2"
    assert d2 == d1


@pytest.mark.parametrize("b,s,t", [(1, 1, 1), (1, 1, 4096), (128, 2, 5000)])
def test_second_order2_vs_order3_printed(b, s, t):
    g = GOLD["second_order2_minus_order3"]
    d = _flops(2, b, s, t, "second", with_o=True) - _flops(3, b, s, t, "second")
    assert d == g["slope_bs"] * b * s + g["intercept"]


def test_absorbed_attention_mac_count_printed():
    """izhida.com: 128 x (512+64+512) x 4K = 557056K = 544M MAC per layer; x60 = 31.875G."""
    g = GOLD["absorbed_attention_macs"]
    c = O.step_flops(2, 1, 1, g["T"], h=g["h"], R=g["R"])
    macs = c.total("qk_lat", "qk_rope", "pv_lat") // 2
    assert macs == g["printed_kilo"] * 1024
    assert macs == g["printed_mega"] * 2 ** 20
    assert macs * g["layers"] == int(g["printed_giga_all_layers"] * 2 ** 30)


def test_cache_and_weight_sizes_printed():
    assert O.D_C + O.D_ROPE == GOLD["cache_row"]["elements"]
    g = GOLD["kv_bytes_per_token"]
    assert g["layers"] * (O.D_C + O.D_ROPE) * 2 == g["bytes"]
    assert O.N_HEADS * O.D_C * O.D_NOPE == 2 ** GOLD["factored_weight_elements"]["w_uk_elements_log2"]


def test_decode_counter_matches_step_counts():
    """The decode oracle charges exactly the order-1 step counts per sequence."""
    rng = np.random.default_rng(5)
    h, d, R, k, v, T = 3, 4, 2, 8, 5, 7
    cache = [rng.standard_normal((T, k + R))]
    c = O.FlopCounter()
    O.mla_decode(rng.standard_normal((1, h, d)), rng.standard_normal((1, h, R)), cache,
                 rng.standard_normal((k, h, d)), rng.standard_normal((k, h, v)), 1, counter=c, chunk=3)
    ref = O.step_flops(1, 1, 1, T, h=h, d=d, k=k, v=v, R=R)
    for label in ("uk", "qk", "qk_rope", "uv", "pv"):
        assert c.terms[label] == ref.terms[label], label


# ---------------------------------------------------------------- algebra
def _tiny(rng, b=2, s=3, t=5, h=4, d=6, k=10, q=7, v=5, e=9):
    return dict(cQ=rng.standard_normal((b, s, q)), W_UQ=rng.standard_normal((q, h, d)),
                W_UK=rng.standard_normal((k, h, d)), ckv=rng.standard_normal((b, t, k)),
                W_UV=rng.standard_normal((k, h, v)), W_O=rng.standard_normal((h, v, e)),
                score=rng.random((b, h, s, t)))


def test_first_absorption_orders_agree():
    x = _tiny(np.random.default_rng(0))
    r = [O.first_absorption_logits(o, x["cQ"], x["W_UK"], x["ckv"], W_UQ=x["W_UQ"]) for o in (1, 2, 3)]
    for a in r[1:]:
        np.testing.assert_allclose(a, r[0], rtol=1e-12, atol=1e-11)


def test_second_absorption_orders_agree():
    x = _tiny(np.random.default_rng(1))
    r = [O.second_absorption_output(o, x["score"], x["ckv"], x["W_UV"], W_O=x["W_O"]) for o in (1, 2, 3)]
    for a in r[1:]:
        np.testing.assert_allclose(a, r[0], rtol=1e-12, atol=1e-11)


def test_first_absorption_matches_textbook_definition():
    """Order 1 equals the plain product (W^UQ c^Q)^T (W^UK c^KV) written with matmuls per head."""
    x = _tiny(np.random.default_rng(2))
    got = O.first_absorption_logits(1, x["cQ"], x["W_UK"], x["ckv"], W_UQ=x["W_UQ"])
    b, s, q = x["cQ"].shape
    k, h, d = x["W_UK"].shape
    for bi in range(b):
        for hi in range(h):
            Q = x["cQ"][bi] @ x["W_UQ"][:, hi, :]          # (s, d)
            K = x["ckv"][bi] @ x["W_UK"][:, hi, :]         # (t, d)
            np.testing.assert_allclose(got[bi, hi], Q @ K.T, rtol=1e-12, atol=1e-11)


def _rand_decode(rng, B, s_q, H, d, R, k, v, lens):
    caches = [rng.standard_normal((T, k + R)) for T in lens]
    return (rng.standard_normal((B * s_q, H, d)), rng.standard_normal((B * s_q, H, R)), caches,
            rng.standard_normal((k, H, d)) / math.sqrt(k), rng.standard_normal((k, H, v)) / math.sqrt(k))


@pytest.mark.parametrize("s_q,lens", [(1, [1, 7, 33]), (2, [2, 5, 40]), (2, [3])])
def test_decode_order1_equals_absorbed(s_q, lens):
    rng = np.random.default_rng(3)
    args = _rand_decode(rng, len(lens), s_q, 5, 8, 4, 16, 6, lens)
    ref = O.mla_decode(*args, s_q, chunk=4)
    ab = O.mla_decode_absorbed(*args, s_q)
    np.testing.assert_allclose(ab, ref["out"], rtol=1e-12, atol=1e-12)
    # the order-2 intermediates reproduce the output through W^UV
    out2 = np.einsum("nhk,khv->nhv", ref["o_lat"], args[4])
    np.testing.assert_allclose(out2, ref["out"], rtol=1e-12, atol=1e-12)
    ql = np.einsum("nhd,khd->nhk", args[0], args[3])
    np.testing.assert_allclose(ref["q_lat"], ql, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("s_q,T", [(1, 1), (1, 3), (1, 5), (2, 3), (2, 5), (2, 2), (4, 4), (3, 5)])
def test_decode_matches_brute_force(s_q, T):
    rng = np.random.default_rng(10 + T + s_q)
    B, H, d, R, k, v = 2, 2, 4, 2, 8, 4
    args = _rand_decode(rng, B, s_q, H, d, R, k, v, [T, T + 1])
    scale = 1 / math.sqrt(d + R)
    ref = O.mla_decode(*args, s_q, scale=scale, chunk=2)
    out, lse = brute_decode(args[0].tolist(), args[1].tolist(), [c.tolist() for c in args[2]],
                            args[3].tolist(), args[4].tolist(), s_q, scale)
    np.testing.assert_allclose(ref["out"], np.array(out), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(ref["lse"], np.array(lse), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- softmax
def test_masked_softmax_matches_scipy():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((3, 4, 50)) * 5
    keep = np.ones_like(x, dtype=bool)
    keep[..., 37:] = False
    p, lse = O.masked_softmax(x, keep)
    np.testing.assert_allclose(p[..., :37], scipy.special.softmax(x[..., :37], axis=-1), rtol=1e-13)
    assert np.all(p[..., 37:] == 0)
    np.testing.assert_allclose(lse, scipy.special.logsumexp(x[..., :37], axis=-1), rtol=1e-13)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-12)


def test_default_scale_is_inverse_sqrt_192():
    assert O.default_scale() == 1 / math.sqrt(192)


# ---------------------------------------------------------------- closed forms
def test_single_token_output_is_value_up_projection():
    """T = 1: the only weight is 1, so out = W^UV^T c_0 for every head and query."""
    rng = np.random.default_rng(6)
    qn, qr, caches, W_UK, W_UV = _rand_decode(rng, 1, 1, 4, 8, 4, 16, 6, [1])
    out = O.mla_decode(qn, qr, caches, W_UK, W_UV, 1)["out"][0]
    c0 = caches[0][0, :16]
    for h in range(4):
        np.testing.assert_allclose(out[h], W_UV[:, h, :].T @ c0, rtol=1e-13, atol=1e-14)


def test_identical_rows_give_value_for_any_query():
    rng = np.random.default_rng(7)
    qn, qr, caches, W_UK, W_UV = _rand_decode(rng, 1, 1, 3, 8, 4, 16, 6, [9])
    caches = [np.tile(caches[0][:1], (9, 1))]
    out = O.mla_decode(qn * 40, qr, caches, W_UK, W_UV, 1)["out"][0]
    c0 = caches[0][0, :16]
    for h in range(3):
        np.testing.assert_allclose(out[h], W_UV[:, h, :].T @ c0, rtol=1e-12, atol=1e-13)


def test_zero_query_gives_mean_value():
    rng = np.random.default_rng(8)
    qn, qr, caches, W_UK, W_UV = _rand_decode(rng, 1, 1, 3, 8, 4, 16, 6, [11])
    res = O.mla_decode(qn * 0, qr * 0, caches, W_UK, W_UV, 1)
    mean_c = caches[0][:, :16].mean(0)
    for h in range(3):
        np.testing.assert_allclose(res["out"][0, h], W_UV[:, h, :].T @ mean_c, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(res["lse"], math.log(11), rtol=1e-13)


def test_two_token_rope_weight_closed_form():
    """q_nope = 0; q_rope . (k_rope_1 - k_rope_0) = sqrt(192) ln 3, so the weights are 1/4, 3/4.

    Fixes the scale 1/sqrt(192), the sign of the RoPE score and that it is added.
    """
    H, d, R, k, v = 2, 128, 64, 512, 128
    rng = np.random.default_rng(9)
    cache = np.zeros((2, k + R))
    cache[:, :k] = rng.standard_normal((2, k))
    cache[1, k] = 1.0                      # k_rope_1 = e_0, k_rope_0 = 0
    qr = np.zeros((1, H, R))
    qr[0, :, 0] = math.sqrt(192) * math.log(3)
    W_UK = rng.standard_normal((k, H, d))
    W_UV = rng.standard_normal((k, H, v))
    out = O.mla_decode(np.zeros((1, H, d)), qr, [cache], W_UK, W_UV, 1)["out"][0]
    V0 = np.einsum("k,khv->hv", cache[0, :k], W_UV)
    V1 = np.einsum("k,khv->hv", cache[1, :k], W_UV)
    np.testing.assert_allclose(out, 0.25 * V0 + 0.75 * V1, rtol=1e-12, atol=1e-12)


def test_causal_first_new_token_sees_only_the_past():
    """s = 2, T = 2: query 0 sits at position 0 and sees token 0 alone."""
    rng = np.random.default_rng(11)
    qn, qr, caches, W_UK, W_UV = _rand_decode(rng, 1, 2, 3, 8, 4, 16, 6, [2])
    out = O.mla_decode(qn, qr, caches, W_UK, W_UV, 2)["out"]
    c0 = caches[0][0, :16]
    for h in range(3):
        np.testing.assert_allclose(out[0, h], W_UV[:, h, :].T @ c0, rtol=1e-13, atol=1e-14)


def test_split_merge_by_lse_equals_unsplit():
    """Softmax over [0,T) equals the LSE-weighted merge of any partition's softmaxes."""
    rng = np.random.default_rng(12)
    qn, qr, caches, W_UK, W_UV = _rand_decode(rng, 1, 1, 4, 8, 4, 16, 6, [37])
    full = O.mla_decode(qn, qr, caches, W_UK, W_UV, 1)
    for cuts in ([10], [1, 36], [5, 17, 30]):
        bounds = [0] + cuts + [37]
        outs, lses = [], []
        for a, b in zip(bounds[:-1], bounds[1:]):
            r = O.mla_decode(qn, qr, [caches[0][a:b]], W_UK, W_UV, 1)
            outs.append(r["out"])
            lses.append(r["lse"])
        L = np.logaddexp.reduce(np.stack(lses), axis=0)
        merged = sum(np.exp(l - L)[..., None] * o for o, l in zip(outs, lses))
        np.testing.assert_allclose(merged, full["out"], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(L, full["lse"], rtol=1e-13)


def test_chunking_does_not_change_result():
    rng = np.random.default_rng(13)
    args = _rand_decode(rng, 2, 2, 3, 8, 4, 16, 6, [50, 21])
    a = O.mla_decode(*args, 2, chunk=7)
    b = O.mla_decode(*args, 2, chunk=4096)
    np.testing.assert_allclose(a["out"], b["out"], rtol=1e-13, atol=1e-14)


def test_head_subset_equals_full():
    rng = np.random.default_rng(14)
    args = _rand_decode(rng, 2, 1, 6, 8, 4, 16, 6, [9, 4])
    full = O.mla_decode(*args, 1)
    sub = O.mla_decode(*args, 1, heads=[4, 1])
    for key in ("out", "lse", "q_lat", "o_lat"):
        np.testing.assert_allclose(sub[key], full[key][:, [4, 1]], rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- planted mistakes
def test_planted_mistakes_are_caught(monkeypatch):
    """A dropped RoPE term, a wrong scale or a transposed W^UK each fail a pin above."""
    H, d, R, k, v = 2, 4, 2, 8, 4
    rng = np.random.default_rng(15)
    args = _rand_decode(rng, 1, 1, H, d, R, k, v, [5])
    scale = 1 / math.sqrt(d + R)
    want, _ = brute_decode(args[0].tolist(), args[1].tolist(), [c.tolist() for c in args[2]],
                           args[3].tolist(), args[4].tolist(), 1, scale)
    good = O.mla_decode(*args, 1, scale=scale)["out"]
    assert np.allclose(good, want, rtol=1e-12, atol=1e-13)

    real_rope = O.rope_logits
    monkeypatch.setattr(O, "rope_logits", lambda q, kk, counter=None: 0 * real_rope(q, kk))
    assert not np.allclose(O.mla_decode(*args, 1, scale=scale)["out"], want, rtol=1e-6)
    monkeypatch.setattr(O, "rope_logits", real_rope)

    assert not np.allclose(O.mla_decode(*args, 1, scale=scale * 1.01)["out"], want, rtol=1e-6)

    W_UK_T = args[3].transpose(0, 2, 1).copy() if H == d else args[3][:, ::-1, :].copy()
    bad = O.mla_decode(args[0], args[1], args[2], W_UK_T, args[4], 1, scale=scale)["out"]
    assert not np.allclose(bad, want, rtol=1e-6)
