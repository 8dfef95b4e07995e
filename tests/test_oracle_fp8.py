"""Pins of the FP8 oracle (block quantisation and the block-quantised BMMs)
against things other than itself: torch's float8_e4m3fn cast, the E4M3 format
definition's fixed points, inputs whose quantisation is exact (where the FP8
BMMs must reproduce the plain contractions of the float64 oracle), and
scalar brute force on tiny shapes."""
import numpy as np
import pytest
import torch

from oracle import fp8 as F
from oracle import mla_oracle as O


def test_e4m3_round_matches_torch_cast():
    rng = np.random.default_rng(0)
    mag = np.exp2(rng.uniform(-12, np.log2(448.0), size=20000))
    x = (mag * rng.choice([-1.0, 1.0], size=mag.size)).astype(np.float32)
    # exact ties between neighbours in several binades, and the subnormal range
    e = rng.integers(-9, 8, size=4000)
    m = rng.integers(0, 8, size=4000)
    base = np.where(e >= -6, np.ldexp(1.0 + m / 8.0, np.maximum(e, -6)), np.ldexp(m / 8.0, -6))
    quantum = np.ldexp(1.0, np.maximum(e, -6) - 3)
    ties = (base + quantum / 2).astype(np.float32)
    ties = ties[ties < 448]
    x = np.concatenate([x, ties, -ties, np.float32([0.0, 448.0, -448.0, 2.0 ** -9, 2.0 ** -10])]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = F.e4m3_round(x)
    assert np.array_equal(got, want)


def test_e4m3_decode_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    got = F.e4m3_decode(codes)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    finite = ~np.isnan(want)
    assert np.array_equal(np.isnan(got), ~finite)
    assert np.array_equal(got[finite], want[finite])
    assert np.nanmax(got) == 448.0 and np.nanmin(got) == -448.0
    # every finite code is a fixed point of the rounding
    assert np.array_equal(F.e4m3_round(got[finite]), got[finite])
    assert sorted(set(np.abs(got[finite]).tolist()))[1] == 2.0 ** -9     # smallest subnormal


@pytest.mark.parametrize("x,want", [
    (448.0, 448.0), (464.0, 448.0), (1e6, 448.0), (-500.0, -448.0),   # saturation
    (1.0625, 1.0), (1.1875, 1.25),                                      # ties to even mantissa
    (2.0 ** -9, 2.0 ** -9), (2.0 ** -10, 0.0), (3 * 2.0 ** -10, 2.0 ** -8),   # subnormals
    (0.1, 0.1015625), (-3.3, -3.25), (240.0, 240.0), (250.0, 256.0),
])
def test_e4m3_known_values(x, want):
    assert F.e4m3_round(np.float32(x)) == want


def test_quantisation_error_bound():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((64, 3, 512)).astype(np.float32) * np.float32(3.0)
    q, s = F.quantize_act(x)
    assert q.shape == x.shape and s.shape == (64, 3, 4)
    deq = q * np.repeat(s.astype(np.float64), 128, axis=2)
    # half a spacing of the code grid, relative 2^-4, plus the subnormal spacing
    bound = np.abs(x) * 2.0 ** -4 * (1 + 1e-6) + np.repeat(s.astype(np.float64), 128, axis=2) * 2.0 ** -10
    assert np.all(np.abs(deq - x) <= bound)
    # the block maximum lands on the largest code
    assert np.allclose(np.max(np.abs(q.reshape(64, 3, 4, 128)), axis=3), 448.0)
    zq, zs = F.quantize_act(np.zeros((2, 1, 256), np.float32))
    assert np.all(zq == 0) and np.all(zs == 1.0)


def _exact_case(rng, H=3, N=5):
    """Integers in [-7, 7] times a power of two per block, with the magnitude
    7 * 2^j present in every block: the scale 7 * 2^j / 448 = 2^(j - 6) and
    its inverse are exact, so every code is exact."""
    # W_UK [512][H][128]: one 128 x 128 block per (k-block, head)
    wuk = rng.integers(-7, 8, size=(512, H, 128)).astype(np.float64)
    wuv = rng.integers(-7, 8, size=(512, H, 128)).astype(np.float64)
    for kb in range(4):
        for h in range(H):
            j = int(rng.integers(-8, 3))
            wuk[kb * 128:(kb + 1) * 128, h, :] *= 2.0 ** j
            wuk[kb * 128, h, 0] = 7 * 2.0 ** j
            j = int(rng.integers(-8, 3))
            wuv[kb * 128:(kb + 1) * 128, h, :] *= 2.0 ** j
            wuv[kb * 128 + 5, h, 7] = -7 * 2.0 ** j
    q = rng.integers(-7, 8, size=(N, H, 128)).astype(np.float64)
    o = rng.integers(-7, 8, size=(N, H, 512)).astype(np.float64)
    for n in range(N):
        for h in range(H):
            j = int(rng.integers(-4, 4))
            q[n, h] *= 2.0 ** j
            q[n, h, 3] = 7 * 2.0 ** j
            for kb in range(4):
                j = int(rng.integers(-6, 2))
                o[n, h, kb * 128:(kb + 1) * 128] *= 2.0 ** j
                o[n, h, kb * 128 + 9] = 7 * 2.0 ** j
    return wuk, wuv, q, o


def test_fp8_bmms_exact_on_representable_inputs():
    rng = np.random.default_rng(2)
    wuk, wuv, q, o = _exact_case(rng)
    Wq_uk, s_uk = F.quantize_w_uk(wuk)
    Wq_uv, s_uv = F.quantize_w_uv(wuv)
    # quantisation is exact here: codes * scales give the inputs back
    assert np.array_equal(Wq_uk * np.repeat(s_uk, 128, axis=1)[:, :, None], np.transpose(wuk, (1, 0, 2)))
    assert np.array_equal(Wq_uv * np.repeat(s_uv, 128, axis=1)[:, None, :], np.transpose(wuv, (1, 2, 0)))
    got_q = F.absorb_fp8(q, Wq_uk, s_uk)
    want_q = O.contract(None, "absorb_q", "nhd,khd->nhk", q, wuk)
    assert np.allclose(got_q, want_q, rtol=1e-12, atol=0)
    got_o = F.out_uv_fp8(o, Wq_uv, s_uv)
    want_o = O.contract(None, "out_uv", "nhk,khv->nhv", o, wuv)
    assert np.allclose(got_o, want_o, rtol=1e-12, atol=0)


def _brute_quant(vec):
    """One 128-vector, scalar float32 steps of the stated recipe."""
    amax = np.float32(0.0)
    for x in vec:
        amax = max(amax, np.float32(abs(np.float32(x))))
    if amax == 0:
        return [0.0] * len(vec), np.float32(1.0)
    s = np.float32(amax / np.float32(448.0))
    r = np.float32(np.float32(448.0) / amax)
    return [float(F.e4m3_round(np.float32(np.float32(x) * r))) for x in vec], s


def test_fp8_bmms_brute_force():
    rng = np.random.default_rng(3)
    H, N = 2, 3
    wuk = rng.standard_normal((512, H, 128)).astype(np.float32) / np.float32(22.6)
    wuv = rng.standard_normal((512, H, 128)).astype(np.float32) / np.float32(22.6)
    q = rng.standard_normal((N, H, 128)).astype(np.float32)
    o = (rng.standard_normal((N, H, 512)) * 0.05).astype(np.float32)
    Wq_uk, s_uk = F.quantize_w_uk(wuk)
    Wq_uv, s_uv = F.quantize_w_uv(wuv)
    got_q = F.absorb_fp8(q, Wq_uk, s_uk)
    got_o = F.out_uv_fp8(o, Wq_uv, s_uv)
    for h in range(H):
        for kb in range(4):
            blk = wuk[kb * 128:(kb + 1) * 128, h, :]
            amax = np.float32(np.max(np.abs(blk)))
            assert s_uk[h, kb] == np.float32(amax / np.float32(448.0))
            blk = wuv[kb * 128:(kb + 1) * 128, h, :]
            assert s_uv[h, kb] == np.float32(np.float32(np.max(np.abs(blk))) / np.float32(448.0))
    for n in range(N):
        for h in range(H):
            cq, sq = _brute_quant(q[n, h])
            for k in (0, 1, 127, 128, 300, 511):
                acc = 0.0
                for d in range(128):
                    acc += cq[d] * Wq_uk[h, k, d]
                want = acc * float(sq) * float(s_uk[h, k // 128])
                assert abs(got_q[n, h, k] - want) <= 1e-12 * max(1.0, abs(want))
            blocks = [_brute_quant(o[n, h, kb * 128:(kb + 1) * 128]) for kb in range(4)]
            for v in (0, 64, 127):
                total = 0.0
                for kb in range(4):
                    co, so = blocks[kb]
                    acc = 0.0
                    for kk in range(128):
                        acc += co[kk] * Wq_uv[h, v, kb * 128 + kk]
                    total += acc * float(so) * float(s_uv[h, kb])
                assert abs(got_o[n, h, v] - total) <= 1e-12 * max(1.0, abs(total))


def test_fp8_bmm_error_against_bf16_path_is_quantisation_sized():
    """The FP8 products differ from the unquantised ones by the quantisation
    error only: a few percent, not a layout or scale mistake."""
    rng = np.random.default_rng(4)
    H, N = 4, 16
    wuk = (rng.standard_normal((512, H, 128)) / np.sqrt(512)).astype(np.float32)
    wuv = (rng.standard_normal((512, H, 128)) / np.sqrt(512)).astype(np.float32)
    q = rng.standard_normal((N, H, 128)).astype(np.float32)
    o = (rng.standard_normal((N, H, 512)) * 0.05).astype(np.float32)
    Wq_uk, s_uk = F.quantize_w_uk(wuk)
    Wq_uv, s_uv = F.quantize_w_uv(wuv)
    ref_q = O.contract(None, "absorb_q", "nhd,khd->nhk", q.astype(np.float64), wuk.astype(np.float64))
    ref_o = O.contract(None, "out_uv", "nhk,khv->nhv", o.astype(np.float64), wuv.astype(np.float64))
    rel = lambda a, b: np.linalg.norm(a - b) / np.linalg.norm(b)
    eq, eo = rel(F.absorb_fp8(q, Wq_uk, s_uk), ref_q), rel(F.out_uv_fp8(o, Wq_uv, s_uv), ref_o)
    assert 0.005 < eq < 0.06 and 0.005 < eo < 0.06, (eq, eo)


def test_cache_quantisation_pins():
    rng = np.random.default_rng(5)
    # exact case: integers in [-7, 7] times a power of two per block, 7 * 2^j present
    c = rng.integers(-7, 8, size=(9, 512)).astype(np.float64)
    for t in range(9):
        for kb in range(4):
            j = int(rng.integers(-5, 3))
            c[t, kb * 128:(kb + 1) * 128] *= 2.0 ** j
            c[t, kb * 128 + 17] = -7 * 2.0 ** j
    q, s = F.quantize_cache(c)
    assert s.shape == (9, 4)
    assert np.array_equal(F.dequantize_cache(q, s), c)
    # general rows: within half a code spacing, scales from each block's own maximum
    x = (rng.standard_normal((33, 512)) * 2.0).astype(np.float32)
    q, s = F.quantize_cache(x)
    for t in (0, 7, 32):
        for kb in range(4):
            blk = x[t, kb * 128:(kb + 1) * 128]
            assert s[t, kb] == np.float32(np.float32(np.max(np.abs(blk))) / np.float32(448.0))
    err = np.abs(F.dequantize_cache(q, s) - x)
    assert np.all(err <= np.abs(x) * 2.0 ** -4 * (1 + 1e-6) + np.repeat(s, 128, axis=1) * 2.0 ** -10)


def test_attention_over_an_exactly_quantised_cache_is_unchanged():
    """Decode attention over the dequantised cache equals attention over the
    original rows when the quantisation is exact: the cache quantiser changes
    nothing but the stored bytes."""
    rng = np.random.default_rng(6)
    H, T = 4, 70
    W_UK = rng.standard_normal((512, H, 128)) / np.sqrt(512)
    W_UV = rng.standard_normal((512, H, 128)) / np.sqrt(512)
    c = rng.integers(-7, 8, size=(T, 512)).astype(np.float64) * 2.0 ** -3
    c[:, ::128] = 7 * 2.0 ** -3                            # every block holds its scale's maximum
    k_rope = rng.standard_normal((T, 64))
    q_nope = rng.standard_normal((1, H, 128))
    q_rope = rng.standard_normal((1, H, 64))
    codes, s = F.quantize_cache(c)
    row = lambda ckv: np.concatenate([ckv, k_rope], axis=1)
    a = O.mla_decode(q_nope, q_rope, [row(c)], W_UK, W_UV, 1, with_intermediates=False)["out"]
    b = O.mla_decode(q_nope, q_rope, [row(F.dequantize_cache(codes, s))], W_UK, W_UV, 1,
                     with_intermediates=False)["out"]
    assert np.array_equal(a, b)
