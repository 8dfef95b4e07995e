"""FP8 block quantisation and the block-quantised projection BMMs -- TEST
INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
legs may import this module.  It shares no code with the CUDA path.

What it computes
----------------
"Lower latency and higher throughput with multi-node DeepSeek deployment"
(Perplexity), section "Quantization": DeepSeek-V3/R1 weights are quantised
statically and activations on the fly; the scaling factors belong to vectors
of 128 elements for activations and to 128 x 128 blocks for weight matrices,
so an (M, K) x (K, N) layer carries activation scales of shape
M x ceil(K / 128) and weight scales of shape ceil(K / 128) x ceil(N / 128).
Section "MLA layer": kv_b_proj is split into k_b_proj and v_b_proj, and both
run as FP8 block-quantised BMMs.  In the absorbed decode path those are

  absorb  : q_lat[n,h,k] = sum_d q_nope[n,h,d] W_UK[k,h,d]   (K = d = 128)
  out_uv  : out[n,h,v]   = sum_k o_lat[n,h,k]  W_UV[k,h,v]   (K = k = 512)

one (M, K) x (K, N) product per head h, with the tokens as M.

Readings where the pages are silent:
  * the FP8 format is E4M3 in its "FN" form: 4 exponent bits with bias 7, 3
    mantissa bits, no infinities, largest finite value 448, subnormals down
    to 2^-9;
  * a block's scale is s = amax / 448 in float32 (amax = largest magnitude of
    the block), so that amax maps to the largest finite code; an all-zero
    block takes s = 1;
  * a value's code is E4M3(x * r), rounded to nearest-even and saturated at
    +-448, with r = 448 / amax computed once per block in float32 and the
    product x * r rounded to float32 (a multiply, not a division per
    element); an all-zero block takes r = 1;
  * the product of a K-block is the exact sum of code products, scaled by
    s_act * s_weight; the K-blocks' results are summed.  Here everything
    after the codes is float64.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
BLOCK = 128


def e4m3_round(x) -> np.ndarray:
    """Round float values to the nearest E4M3 value (ties to even), saturating
    at +-448.  Returns the represented values as float64.

    From the format definition: a normal value is 2^(E-7) (1 + m/8) with
    E in 1..15 (and E = 15, m = 7 reserved for NaN, hence the 448 limit); a
    subnormal is 2^-6 (m/8).  So the spacing of representable values is
    2^(e-3) in the binade [2^e, 2^(e+1)) for e >= -6 and 2^-9 below 2^-6.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    # exponent of the binade: a = f * 2^e2 with f in [0.5, 1)  ->  e = e2 - 1
    _, e2 = np.frexp(np.where(a > 0, a, 1.0))
    e = np.maximum(e2.astype(np.int64) - 1, -6)          # below 2^-6: subnormal spacing
    quantum = np.ldexp(1.0, e - 3)
    r = np.rint(a / quantum) * quantum                    # np.rint: ties to even; exact in float64
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Bytes (uint8) of E4M3 codes -> float64 values, from the format
    definition (NaN for the reserved S.1111.111 patterns)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    E = (c >> 3) & 0xF
    m = c & 0x7
    normal = np.ldexp(1.0 + m / 8.0, E - 7)
    sub = np.ldexp(m / 8.0, -6)
    v = np.where(E == 0, sub, normal)
    v = np.where((E == 15) & (m == 7), np.nan, v)
    return sign * v


def quantize_blocks(x, axis_blocks: tuple) -> tuple:
    """Block quantisation of a float32 array.

    ``axis_blocks`` gives, per axis, the block length along it (1 = every
    index its own block; the axis length must be a multiple).  Returns
    (codes as float64 values, scales s as float32 with one entry per block,
    shaped like x with every blocked axis divided by its block length).
    """
    x = np.asarray(x, dtype=np.float32)
    assert x.ndim == len(axis_blocks)
    shp = []
    for n, b in zip(x.shape, axis_blocks):
        assert n % b == 0, (n, b)
        shp += [n // b, b]
    xb = x.reshape(shp)
    inner = tuple(range(1, 2 * x.ndim, 2))
    amax = np.max(np.abs(xb), axis=inner, keepdims=True).astype(np.float32)
    nz = amax > 0
    s = np.where(nz, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    r = np.where(nz, np.float32(E4M3_MAX) / np.where(nz, amax, np.float32(1.0)), np.float32(1.0)).astype(np.float32)
    y = (xb * r).astype(np.float32)                       # one float32 multiply per element
    q = e4m3_round(y).reshape(x.shape)
    return q, np.squeeze(s, axis=inner)


def quantize_w_uk(W_UK) -> tuple:
    """W_UK [k=512][h][d=128] -> codes [h][k][d] and scales [h][k/128]
    (one scale per 128 x 128 block of each head's 512 x 128 matrix)."""
    w = np.transpose(np.asarray(W_UK, dtype=np.float32), (1, 0, 2))     # [h][k][d]
    q, s = quantize_blocks(w, (1, BLOCK, BLOCK))
    return q, s.reshape(w.shape[0], -1)


def quantize_w_uv(W_UV) -> tuple:
    """W_UV [k=512][h][v=128] -> codes [h][v][k] and scales [h][k/128]
    (one scale per 128 x 128 block; v = 128 is a single block)."""
    w = np.transpose(np.asarray(W_UV, dtype=np.float32), (1, 2, 0))     # [h][v][k]
    q, s = quantize_blocks(w, (1, BLOCK, BLOCK))
    return q, s.reshape(w.shape[0], -1)


def quantize_act(x) -> tuple:
    """Activations [n][h][K] -> codes and scales [n][h][K/128] (one scale per
    128-element vector along K)."""
    x = np.asarray(x, dtype=np.float32)
    return quantize_blocks(x, (1, 1, BLOCK))


def absorb_fp8(q_nope, Wq_uk, s_uk) -> np.ndarray:
    """q_lat[n,h,k] = s_q[n,h] s_uk[h, k//128] sum_d code(q)[n,h,d] Wq_uk[h,k,d]
    (K = 128 is one block).  float64."""
    qq, sq = quantize_act(q_nope)                         # [n][h][128], [n][h][1]
    acc = np.einsum("nhd,hkd->nhk", qq, np.asarray(Wq_uk, dtype=np.float64))
    s_w = np.repeat(np.asarray(s_uk, dtype=np.float64), BLOCK, axis=1)        # [h][512]
    return acc * sq.astype(np.float64)[:, :, :1] * s_w[None, :, :]


def out_uv_fp8(o_lat, Wq_uv, s_uv) -> np.ndarray:
    """out[n,h,v] = sum_kb s_o[n,h,kb] s_uv[h,kb] sum_{k in kb} code(o)[n,h,k] Wq_uv[h,v,k].
    float64."""
    oq, so = quantize_act(o_lat)                          # [n][h][512], [n][h][4]
    n, h, K = oq.shape
    nkb = K // BLOCK
    Wq = np.asarray(Wq_uv, dtype=np.float64).reshape(h, -1, nkb, BLOCK)       # [h][v][kb][128]
    part = np.einsum("nhbk,hvbk->nhbv", oq.reshape(n, h, nkb, BLOCK), Wq)      # per K-block sums
    scale = so.astype(np.float64) * np.asarray(s_uv, dtype=np.float64)[None, :, :]   # [n][h][kb]
    return np.einsum("nhbv,nhb->nhv", part, scale)


def quantize_cache(ckv) -> tuple:
    """Latent cache rows c_KV [T][512] -> codes [T][512] and scales [T][4]: one
    scale per 128-element block of each token's row, as for any activation
    ("Quantization": activations carry a scale per 128-element vector).

    Reading: only c_KV is quantised; the 64-wide k_rope part of a cache row
    stays bf16 (the pages quantise GEMM operands by 128-blocks and say nothing
    of the RoPE key, whose 128 bytes are a ninth of the row)."""
    c = np.asarray(ckv, dtype=np.float32)
    assert c.ndim == 2 and c.shape[1] % BLOCK == 0
    return quantize_blocks(c, (1, BLOCK))


def dequantize_cache(codes, scales) -> np.ndarray:
    """codes [T][512] (values) and scales [T][4] -> float64 rows codes * scale."""
    q = np.asarray(codes, dtype=np.float64)
    s = np.repeat(np.asarray(scales, dtype=np.float64), BLOCK, axis=1)
    return q * s
