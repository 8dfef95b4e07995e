"""Float64 CPU oracle of MLA decode attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
legs may import this module.  It shares no code with the CUDA path.

What it computes
----------------
Multi-head Latent Attention (MLA) as the MLA matrix-absorption notes write it
("MLA Matrix Absorption Analysis", wkq9411.github.io):

* first absorption, §2 ("MLA 第一次矩阵吸收的计算量分析"): the attention
  logits (W^UQ c^Q)^T (W^UK c^KV), evaluated in three orders --
  order 1 (§2.1, original: up-project K explicitly), order 2 (§2.2, the
  absorption used in the MLA source: fold W^UK into the query first),
  order 3 (§2.3, pre-absorption: materialise W^UQ^T W^UK);
* second absorption, §3 ("MLA 第二次矩阵吸收的计算量分析"): the output
  W^O [score (W^UV c^KV)], again in three orders (§3.1, §3.2, §3.3).

Tensor shapes follow the notes' symbols (§2.1, §3.1):
  c^Q (b,s,q); W^UQ (q,h,d); W^UK (k,h,d); c^KV (b,t,k);
  score (b,h,s,t); W^UV (k,h,v); W^O (h,v,e).

The decoupled RoPE key is the extra MQA term of "How is DeepSeek-V2's
inference cost computed?" (izhida.com, the expert answer): one RoPE'd key of
width 64 shared by all heads, whose q.k score is *added* to the latent score.
q_rope and k_rope arrive already rotated; no rotation happens here.

Readings where the pages are silent:
  * softmax scale = 1/sqrt(d_nope + d_rope) = 1/sqrt(192), no extra factor;
  * the softmax is the standard one over the key axis t;
  * the s new tokens are already in the cache: query i of s sits at position
    T - s + i and attends keys t <= T - s + i (causal among the new tokens).

FLOP convention
---------------
Every contraction goes through :func:`contract`, which adds 2 * (product of
all index extents) to a labelled counter: one multiply-add = 2 FLOPs, the
"with bias" convention of the notes' §1.1, under which a contraction's FLOPs
are twice the product of its dimensions.
"""
from __future__ import annotations

import math
from collections import defaultdict
from dataclasses import dataclass

import numpy as np

# Dimensions the pages fix for DeepSeek-V2/V3 (izhida.com answer; notes §2.4, §3.4).
D_NOPE = 128      # d   : qk_nope_head_dim
D_ROPE = 64       # R   : RoPE head dim, "每个head的内积为64维"
D_C = 512         # k   : kv_lora_rank (latent width of c^KV)
D_V = 128         # v   : v_head_dim
D_CQ = 1536       # q   : q_lora_rank (d_c')
N_HEADS = 128     # h
DIM_V3 = 7168     # e   : model dim used in the notes' §3.4 worked numbers


# --------------------------------------------------------------------------
# FLOP counting
# --------------------------------------------------------------------------
class FlopCounter:
    """Labelled FLOP tally; ``dry=True`` counts without doing arithmetic."""

    def __init__(self, dry: bool = False):
        self.dry = dry
        self.terms: dict[str, int] = defaultdict(int)

    def total(self, *labels: str) -> int:
        if not labels:
            return sum(self.terms.values())
        return sum(self.terms[l] for l in labels)


@dataclass(frozen=True)
class Shape:
    """Shape-only stand-in for an array, used by a dry FlopCounter."""
    shape: tuple

    @property
    def ndim(self) -> int:
        return len(self.shape)


def contract(counter: FlopCounter | None, label: str, spec: str, *ops):
    """einsum in float64 that charges 2 * prod(all index extents) FLOPs.

    ``spec`` is an explicit einsum spec ('ab,bc->ac').  With a dry counter the
    operands may be :class:`Shape` objects and a :class:`Shape` is returned.
    """
    lhs, out = spec.split("->")
    ins = lhs.split(",")
    assert len(ins) == len(ops), spec
    extent: dict[str, int] = {}
    for sub, op in zip(ins, ops):
        assert len(sub) == len(op.shape), (spec, sub, op.shape)
        for ch, n in zip(sub, op.shape):
            if ch in extent and extent[ch] != n:
                raise ValueError(f"extent mismatch for '{ch}' in {spec}: {extent[ch]} vs {n}")
            extent[ch] = int(n)
    if counter is not None:
        counter.terms[label] += 2 * math.prod(extent.values())
    if counter is not None and counter.dry:
        return Shape(tuple(extent[ch] for ch in out))
    return np.einsum(spec, *[np.asarray(o, dtype=np.float64) for o in ops], optimize=True)


# --------------------------------------------------------------------------
# First absorption: the nope part of the logits, (b, h, s, t)
# --------------------------------------------------------------------------
def first_absorption_logits(order: int, q_in, W_UK, ckv, W_UQ=None, counter=None):
    """Latent ("nope") attention logits (W^UQ c^Q)^T (W^UK c^KV), shape (b,h,s,t).

    ``q_in`` is c^Q (b,s,q) when ``W_UQ`` is given, else the up-projected
    q_nope (b,s,h,d) and Step 1 is skipped.  Orders follow the notes:

    order 1 (§2.1): Step 2 K = W^UK c^KV (b,t,h,d); Step 3 q.K.
    order 2 (§2.2): Step 2 q^T W^UK (b,s,h,k); Step 3 that . c^KV.
    order 3 (§2.3): Step 1 W^UQ^T W^UK (h,q,k); Step 2 c^Q . that; Step 3 . c^KV.

    Labels: 'uq' (2bshdq), 'uk' (2bthdk), 'qk' (2bhstd), 'absorb_q'
    (2bshkd), 'qk_lat' (2bhstk), 'pre_uq_uk' (2hqkd), 'cq_pre' (2bshkq).
    Pinned by the notes' printed differences (§2.4.1, §2.4.2) and by
    order agreement / brute force in tests.
    """
    if order == 3:
        if W_UQ is None:
            raise ValueError("order 3 needs c^Q and W^UQ")
        Wqk = contract(counter, "pre_uq_uk", "qhd,khd->hqk", W_UQ, W_UK)
        qc = contract(counter, "cq_pre", "bsq,hqk->bshk", q_in, Wqk)
        return contract(counter, "qk_lat", "bshk,btk->bhst", qc, ckv)
    if W_UQ is not None:
        q_nope = contract(counter, "uq", "bsq,qhd->bshd", q_in, W_UQ)
    else:
        q_nope = q_in
    if order == 1:
        K = contract(counter, "uk", "btk,khd->bthd", ckv, W_UK)
        return contract(counter, "qk", "bshd,bthd->bhst", q_nope, K)
    if order == 2:
        q_lat = contract(counter, "absorb_q", "bshd,khd->bshk", q_nope, W_UK)
        return contract(counter, "qk_lat", "bshk,btk->bhst", q_lat, ckv)
    raise ValueError(f"order must be 1, 2 or 3, got {order}")


# --------------------------------------------------------------------------
# Second absorption: the attention output, (b, h, s, v) or (b, h, s, e)
# --------------------------------------------------------------------------
def second_absorption_output(order: int, score, ckv, W_UV, W_O=None, counter=None):
    """Attention output W^O [score (W^UV c^KV)] in the notes' three orders.

    ``score`` is the (already normalised) weight tensor (b,h,s,t).  Without
    ``W_O`` the result is the per-head value output (b,h,s,v) and Step 3 is
    skipped (order 3 needs W_O).

    order 1 (§3.1): Step 1 V = W^UV c^KV (b,t,h,v); Step 2 score.V.
    order 2 (§3.2): Step 1 score.c^KV (b,h,s,k); Step 2 W^UV applied per head.
    order 3 (§3.3): Step 1 W^O W^UV (h,k,e); Step 2 score.c^KV; Step 3.

    Labels: 'uv' (2bthvk), 'pv' (2bhsvt), 'o' (2bhsev), 'pv_lat' (2bhskt),
    'out_uv' (2bhsvk), 'pre_o_uv' (2hkev), 'o_pre' (2bhsek).
    """
    if order == 1:
        V = contract(counter, "uv", "btk,khv->bthv", ckv, W_UV)
        out = contract(counter, "pv", "bhst,bthv->bhsv", score, V)
    elif order == 2:
        o_lat = contract(counter, "pv_lat", "bhst,btk->bhsk", score, ckv)
        out = contract(counter, "out_uv", "bhsk,khv->bhsv", o_lat, W_UV)
    elif order == 3:
        if W_O is None:
            raise ValueError("order 3 needs W^O")
        Wov = contract(counter, "pre_o_uv", "khv,hve->hke", W_UV, W_O)
        o_lat = contract(counter, "pv_lat", "bhst,btk->bhsk", score, ckv)
        return contract(counter, "o_pre", "bhsk,hke->bhse", o_lat, Wov)
    else:
        raise ValueError(f"order must be 1, 2 or 3, got {order}")
    if W_O is not None:
        out = contract(counter, "o", "bhsv,hve->bhse", out, W_O)
    return out


def query_up(c_q, W_UQ, d_nope: int = D_NOPE, counter=None):
    """Per-head queries from the query latent: q = W^UQ applied to c^Q.

    ``c_q`` (n, q) and ``W_UQ`` (q, h, d + R), the notes' W^UQ (q, h, d) of
    section 2.1 extended by the head's RoPE query columns (DeepSeek's q_b_proj
    produces both).  Returns (q_nope (n, h, d), q_rope (n, h, R)); the RoPE
    part is returned before rotation.  Label 'uq' (2 n q h (d + R)).
    """
    q = contract(counter, "uq", "nq,qhf->nhf", c_q, W_UQ)
    if isinstance(q, Shape):   # dry run: shapes only
        n, h, f = q.shape
        return Shape((n, h, d_nope)), Shape((n, h, f - d_nope))
    return q[:, :, :d_nope], q[:, :, d_nope:]


def qkv_down(x, W_DQ, W_DKV, counter=None):
    """The two down-projections of a token's hidden state, as the Perplexity
    write-up's fused qkv_a_proj computes them in one product (section "MLA
    layer": q_a_proj and kv_a_proj merged): c^Q = x W^DQ (n, q) and the
    cache row [c^KV | k_rope] = x W^DKV (n, d_c + R), k_rope before rotation.
    ``x`` (n, e), ``W_DQ`` (e, q), ``W_DKV`` (e, d_c + R).  Labels 'dq', 'dkv'."""
    return contract(counter, "dq", "ne,eq->nq", x, W_DQ), contract(counter, "dkv", "ne,ec->nc", x, W_DKV)


def rope_logits(q_rope, k_rope, counter=None):
    """Decoupled-RoPE score q_rope . k_rope, (b,h,s,t); one key shared by all heads.

    The izhida.com answer: RoPE is an extra MQA whose q.k score is added to
    the MLA score.  Label 'qk_rope' (2bhstR).
    """
    return contract(counter, "qk_rope", "bshr,btr->bhst", q_rope, k_rope)


# --------------------------------------------------------------------------
# Softmax with log-sum-exp
# --------------------------------------------------------------------------
def masked_softmax(logits: np.ndarray, keep: np.ndarray):
    """Standard softmax over the last axis restricted to ``keep``.

    Returns (p, lse) with p = exp(x - max) / sum exp(x - max) on kept
    entries (0 elsewhere) and lse = max + log sum exp(x - max) (natural log).
    Every row must keep at least one entry.
    """
    x = np.where(keep, logits, -np.inf)
    m = np.max(x, axis=-1, keepdims=True)
    if not np.all(np.isfinite(m)):
        raise ValueError("a softmax row has no kept entry")
    e = np.where(keep, np.exp(x - m), 0.0)
    z = np.sum(e, axis=-1, keepdims=True)
    return e / z, (m + np.log(z))[..., 0]


def tree_masks(parents) -> list[int]:
    """Visibility bitmasks of a speculative token tree (EAGLE-style drafts).

    The Perplexity write-up ("Будущая работа" / future work) names EAGLE-style
    speculative decoding that drafts several tokens as a tree.  The pages do
    not write the attention mask out; the plain reading, used here: draft
    token i sees the committed prefix, every ancestor of i in the tree, and
    itself.  ``parents[i]`` is the index of token i's parent among the drafts
    (< i), or -1 when its parent is the last committed token.  Bit j of the
    result's entry i is set iff draft j is visible to draft i.  A chain
    (parents = [-1, 0, 1, ...]) gives the causal masks, a star (all -1) lets
    every draft see only itself.
    """
    masks = []
    for i, par in enumerate(parents):
        if not -1 <= par < i:
            raise ValueError(f"parent of draft {i} must be in [-1, {i})")
        m = 1 << i
        if par >= 0:
            m |= masks[par]
        masks.append(m)
    return masks


def default_scale(d_nope: int = D_NOPE, d_rope: int = D_ROPE) -> float:
    """1/sqrt(d_nope + d_rope): the plain reading for the unstated scale."""
    return 1.0 / math.sqrt(d_nope + d_rope)


# --------------------------------------------------------------------------
# The decode oracle
# --------------------------------------------------------------------------
def mla_decode(q_nope, q_rope, caches, W_UK, W_UV, s_q: int, scale: float | None = None,
               heads=None, chunk: int = 2048, counter: FlopCounter | None = None,
               with_intermediates: bool = True, draft_masks=None):
    """Un-absorbed (order 1) MLA decode attention over per-sequence caches.

    Arguments (all converted to float64):
      q_nope  (N, h, d)   N = B * s_q, row n = b * s_q + i
      q_rope  (N, h, R)
      caches  list of B arrays (T_b, d_c + R): row t = [c^KV_t | k_rope_t]
      W_UK    (d_c, h, d), W_UV (d_c, h, v)   (layouts of the notes' §2.1, §3.1)
      heads   optional subset of head indices (outputs are for those heads)

    Per sequence b, query i and head h (order 1 of both absorptions):
      K = W^UK c^KV, V = W^UV c^KV                         (§2.1 Step 2, §3.1 Step 1)
      logit[t] = scale * (q_nope . K_t + q_rope . k_rope_t) (RoPE-MQA score added)
      keep t <= T_b - s_q + i;  p = softmax(logit)         (standard softmax)
      out = sum_t p[t] V_t                                  (§3.1 Step 2)

    ``draft_masks`` (optional, one list of s_q bitmasks per sequence, e.g.
    from :func:`tree_masks`) replaces the causal rule among the s_q new
    tokens: query i keeps every prefix key t < T_b - s_q and new token j
    (key T_b - s_q + j) iff bit j of draft_masks[b][i] is set.

    Returns a dict with 'out' (N,h',v), 'lse' (N,h') natural-log LSE of the
    scaled logits, and (if ``with_intermediates``) the order-2 intermediates
    'q_lat' = q_nope^T W^UK (N,h',d_c) (§2.2 Step 2) and 'o_lat' = p . c^KV
    (N,h',d_c) (§3.2 Step 1), each computed on its own.  K and V are formed
    in token chunks of ``chunk`` rows; chunking only reorders float64 sums.
    """
    q_nope = np.asarray(q_nope, dtype=np.float64)
    q_rope = np.asarray(q_rope, dtype=np.float64)
    W_UK = np.asarray(W_UK, dtype=np.float64)
    W_UV = np.asarray(W_UV, dtype=np.float64)
    if heads is not None:
        heads = np.asarray(heads, dtype=np.int64)
        q_nope, q_rope = q_nope[:, heads], q_rope[:, heads]
        W_UK, W_UV = W_UK[:, heads], W_UV[:, heads]
    N, H, d = q_nope.shape
    d_c = W_UK.shape[0]
    R = q_rope.shape[2]
    v = W_UV.shape[2]
    B = len(caches)
    if N != B * s_q:
        raise ValueError(f"N={N} rows but B*s_q={B * s_q}")
    if scale is None:
        scale = default_scale(d, R)

    out = np.zeros((N, H, v))
    lse = np.zeros((N, H))
    q_lat = np.zeros((N, H, d_c)) if with_intermediates else None
    o_lat = np.zeros((N, H, d_c)) if with_intermediates else None

    for b in range(B):
        cache = np.asarray(caches[b], dtype=np.float64)
        T = cache.shape[0]
        if T < s_q:
            raise ValueError(f"sequence {b}: T={T} < s_q={s_q}")
        ckv, krope = cache[:, :d_c], cache[:, d_c:d_c + R]
        rows = slice(b * s_q, (b + 1) * s_q)
        qn = q_nope[rows][None]            # (1, s, h, d)
        qr = q_rope[rows]                  # (s, h, R)

        logits = np.empty((H, s_q, T))
        for t0 in range(0, T, chunk):
            t1 = min(T, t0 + chunk)
            part = first_absorption_logits(1, qn, W_UK, ckv[None, t0:t1], counter=counter)
            logits[:, :, t0:t1] = part[0]
        logits += rope_logits(qr[None], krope[None], counter=counter)[0]
        logits *= scale

        pos = np.arange(T)
        if draft_masks is None:
            keep = pos[None, :] <= (T - s_q + np.arange(s_q))[:, None]  # (s, T): causal
        else:
            keep = np.ones((s_q, T), dtype=bool)                         # prefix: all visible
            for i in range(s_q):
                for j in range(s_q):
                    keep[i, T - s_q + j] = bool((int(draft_masks[b][i]) >> j) & 1)
        p, l = masked_softmax(logits, keep[None, :, :])                  # (h, s, T)

        acc = np.zeros((1, H, s_q, v))
        for t0 in range(0, T, chunk):
            t1 = min(T, t0 + chunk)
            acc += second_absorption_output(1, p[None, :, :, t0:t1], ckv[None, t0:t1], W_UV,
                                            counter=counter)
        out[rows] = acc[0].transpose(1, 0, 2)
        lse[rows] = l.T

        if with_intermediates:
            q_lat[rows] = contract(None, "absorb_q", "shd,khd->shk", q_nope[rows], W_UK)
            o_lat[rows] = contract(None, "pv_lat", "hst,tk->shk", p, ckv)

    res = {"out": out, "lse": lse}
    if with_intermediates:
        res["q_lat"] = q_lat
        res["o_lat"] = o_lat
    return res


def mla_decode_absorbed(q_nope, q_rope, caches, W_UK, W_UV, s_q: int, scale: float | None = None,
                        counter: FlopCounter | None = None):
    """Order-2 (absorbed) evaluation of the same decode attention, float64.

    q_lat = q_nope^T W^UK (§2.2 Step 2); logit = scale (q_lat . c^KV +
    q_rope . k_rope) (§2.2 Step 3 plus the RoPE-MQA term); o_lat = p . c^KV
    (§3.2 Step 1); out = W^UV o_lat per head (§3.2 Step 2).  Used to pin the
    order-1 oracle by associativity; the kernels follow this order.
    """
    q_nope = np.asarray(q_nope, dtype=np.float64)
    q_rope = np.asarray(q_rope, dtype=np.float64)
    W_UK = np.asarray(W_UK, dtype=np.float64)
    W_UV = np.asarray(W_UV, dtype=np.float64)
    N, H, d = q_nope.shape
    d_c = W_UK.shape[0]
    R = q_rope.shape[2]
    if scale is None:
        scale = default_scale(d, R)
    out = np.zeros((N, H, W_UV.shape[2]))
    for b, cache in enumerate(caches):
        cache = np.asarray(cache, dtype=np.float64)
        T = cache.shape[0]
        ckv, krope = cache[:, :d_c], cache[:, d_c:d_c + R]
        rows = slice(b * s_q, (b + 1) * s_q)
        logits = first_absorption_logits(2, q_nope[rows][None], W_UK, ckv[None], counter=counter)[0]
        logits = logits + rope_logits(q_rope[rows][None], krope[None], counter=counter)[0]
        logits = logits * scale
        keep = np.arange(T)[None, :] <= (T - s_q + np.arange(s_q))[:, None]
        p, _ = masked_softmax(logits, keep[None])
        o = second_absorption_output(2, p[None], ckv[None], W_UV, counter=counter)[0]
        out[rows] = o.transpose(1, 0, 2)
    return out


# --------------------------------------------------------------------------
# FLOP accounting of the contraction steps (no arithmetic)
# --------------------------------------------------------------------------
def step_flops(order: int, b: int, s: int, t: int, h: int = N_HEADS, d: int = D_NOPE,
               k: int = D_C, v: int = D_V, q: int | None = None, e: int | None = None,
               R: int = 0) -> FlopCounter:
    """Run the contraction steps of one attention in dry mode and return the tally.

    Uses exactly the step functions the oracle computes with
    (:func:`first_absorption_logits`, :func:`rope_logits`,
    :func:`second_absorption_output`) on shape-only operands.  ``q`` adds the
    c^Q / W^UQ input (Step 1 of §2), ``e`` adds W^O (Step 3 of §3), ``R`` > 0
    adds the RoPE-MQA score.  The softmax between the two halves is not a
    contraction and is not counted.
    """
    c = FlopCounter(dry=True)
    ckv = Shape((b, t, k))
    W_UK = Shape((k, h, d))
    if q is not None:
        first_absorption_logits(order, Shape((b, s, q)), W_UK, ckv, W_UQ=Shape((q, h, d)), counter=c)
    else:
        first_absorption_logits(order, Shape((b, s, h, d)), W_UK, ckv, counter=c)
    if R:
        rope_logits(Shape((b, s, h, R)), Shape((b, t, R)), counter=c)
    W_O = Shape((h, v, e)) if e is not None else None
    second_absorption_output(order, Shape((b, h, s, t)), ckv, Shape((k, h, v)), W_O=W_O, counter=c)
    return c
