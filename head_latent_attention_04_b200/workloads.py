"""Seeded synthetic decode workloads (inputs only; none of the method's arithmetic).

This module is the one place both the CUDA path's callers and the CPU oracle's
callers get their inputs from.  It draws random numbers, rounds them to bf16,
lays cache rows out in 64-token pages of a shared pool and writes the block
table.  It computes nothing of MLA itself.

Value distributions: q_nope, q_rope and every cache entry (c^KV and k_rope)
~ N(0, 1); W_UK and W_UV ~ N(0, std 1/sqrt(fan_in)) with fan_in = d_c = 512
(the up-projection direction that consumes c^KV).  All are rounded to bf16.

The five presets are the decode shapes the pages discuss (DeepSeek-V2 heads
and widths; the multi-token-prediction query length 2 of the Perplexity
deployment write-up), see ``PRESETS``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

PAGE = 64
D_NOPE, D_ROPE, D_C, D_V = 128, 64, 512, 128
ROW = D_C + D_ROPE                       # 576 bf16 per cached token
POISON = 8192.0                           # finite, bf16-exact fill of unused pool rows


@dataclass(frozen=True)
class Preset:
    name: str
    B: int
    s_q: int
    n_heads: int
    seed: int
    lens: str              # 'fixed:<T>' | 'uniform:<lo>:<hi>' | 'lognormal:<median>:<sigma>:<cap>'
    pool: str              # 'contiguous' | 'permuted' | 'scattered:<factor>'


PRESETS = {
    "tiny": Preset("tiny", B=2, s_q=1, n_heads=16, seed=0, lens="fixed:256", pool="contiguous"),
    "v2_4k": Preset("v2_4k", B=32, s_q=1, n_heads=128, seed=1, lens="fixed:4096", pool="permuted"),
    "varlen": Preset("varlen", B=64, s_q=1, n_heads=128, seed=2, lens="uniform:512:16384",
                     pool="scattered:1.25"),
    "long128k": Preset("long128k", B=4, s_q=1, n_heads=128, seed=3, lens="fixed:131072",
                       pool="permuted"),
    "mtp2": Preset("mtp2", B=128, s_q=2, n_heads=128, seed=4, lens="lognormal:4096:1.0:32768",
                   pool="permuted"),
}


def draw_seq_lens(spec: str, B: int, s_q: int, rng: np.random.Generator) -> np.ndarray:
    kind, *args = spec.split(":")
    if kind == "fixed":
        T = np.full(B, int(args[0]), dtype=np.int64)
    elif kind == "uniform":
        T = rng.integers(int(args[0]), int(args[1]), size=B, endpoint=True)
    elif kind == "lognormal":
        median, sigma, cap = float(args[0]), float(args[1]), int(args[2])
        T = np.clip(np.rint(rng.lognormal(math.log(median), sigma, size=B)), s_q, cap).astype(np.int64)
    else:
        raise ValueError(spec)
    return T.astype(np.int32)


def _randn_bf16(shape, gen: torch.Generator, device, std: float = 1.0) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


@dataclass
class Workload:
    """One decode batch: queries, weights, a paged latent cache and its page table.

    Layouts (row-major, bf16 unless stated):
      q_nope   [N][h][128]     N = B * s_q, row n = b * s_q + i
      q_rope   [N][h][64]
      w_uk     [512][h][128]   (k, h, d)
      w_uv     [512][h][128]   (k, h, v)
      kv_pool  [num_blocks][64][576]  row = [c^KV (512) | k_rope (64)]
      block_table int32 [B][max_blocks]  (-1 past the last page)
      seq_lens    int32 [B]  (T_b, including the s_q new tokens)
    """
    name: str
    B: int
    s_q: int
    n_heads: int
    seq_lens: np.ndarray
    block_table: np.ndarray
    num_blocks: int
    q_nope: torch.Tensor
    q_rope: torch.Tensor
    w_uk: torch.Tensor
    w_uv: torch.Tensor
    kv_pool: torch.Tensor
    meta: dict = field(default_factory=dict)

    @property
    def N(self) -> int:
        return self.B * self.s_q

    @property
    def max_blocks(self) -> int:
        return int(self.block_table.shape[1])

    @property
    def total_tokens(self) -> int:
        return int(self.seq_lens.astype(np.int64).sum())

    def cache_rows(self, b: int) -> torch.Tensor:
        """Sequence b's cache rows in token order, [T_b][576] (a gather through the page table)."""
        T = int(self.seq_lens[b])
        n_pages = (T + PAGE - 1) // PAGE
        ids = torch.as_tensor(self.block_table[b, :n_pages].astype(np.int64), device=self.kv_pool.device)
        return self.kv_pool.index_select(0, ids).reshape(n_pages * PAGE, ROW)[:T]

    def to(self, device) -> "Workload":
        return Workload(self.name, self.B, self.s_q, self.n_heads, self.seq_lens, self.block_table,
                        self.num_blocks, self.q_nope.to(device), self.q_rope.to(device),
                        self.w_uk.to(device), self.w_uv.to(device), self.kv_pool.to(device),
                        dict(self.meta))


def make_workload(B: int, s_q: int, n_heads: int, seq_lens, seed: int, pool: str = "permuted",
                  device="cpu", name: str = "custom", poison: float = POISON) -> Workload:
    """Draw a seeded decode batch.

    ``pool``: 'contiguous' (sequence pages laid out in order), 'permuted'
    (exactly the pages needed, in a random permutation) or 'scattered:<f>'
    (a pool f times larger, pages at random distinct slots).  Unused pool
    rows and the tail of each sequence's last page hold ``poison``.
    """
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    assert seq_lens.shape == (B,) and np.all(seq_lens >= s_q)
    rng = np.random.default_rng(seed)
    pages = (seq_lens.astype(np.int64) + PAGE - 1) // PAGE
    total_pages = int(pages.sum())
    max_blocks = int(pages.max())

    if pool == "contiguous":
        num_blocks = total_pages
        slots = np.arange(total_pages)
    elif pool == "permuted":
        num_blocks = total_pages
        slots = rng.permutation(total_pages)
    elif pool.startswith("scattered:"):
        num_blocks = int(math.ceil(float(pool.split(":")[1]) * total_pages))
        slots = rng.permutation(num_blocks)[:total_pages]
    else:
        raise ValueError(pool)

    block_table = np.full((B, max_blocks), -1, dtype=np.int32)
    off = 0
    for b in range(B):
        block_table[b, :pages[b]] = slots[off:off + pages[b]]
        off += pages[b]

    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    N = B * s_q
    w_std = 1.0 / math.sqrt(D_C)
    q_nope = _randn_bf16((N, n_heads, D_NOPE), gen, device)
    q_rope = _randn_bf16((N, n_heads, D_ROPE), gen, device)
    w_uk = _randn_bf16((D_C, n_heads, D_NOPE), gen, device, w_std)
    w_uv = _randn_bf16((D_C, n_heads, D_V), gen, device, w_std)

    kv_pool = torch.full((num_blocks, PAGE, ROW), poison, dtype=torch.bfloat16, device=device)
    ids = torch.as_tensor(slots.astype(np.int64), device=device)
    # cache rows in page order, drawn page by page (a 64-row block per page)
    chunk = 4096
    for p0 in range(0, total_pages, chunk):
        p1 = min(total_pages, p0 + chunk)
        kv_pool[ids[p0:p1]] = _randn_bf16((p1 - p0, PAGE, ROW), gen, device)
    # poison the tail of each last page
    for b in range(B):
        tail = int(pages[b] * PAGE - seq_lens[b])
        if tail:
            kv_pool[int(block_table[b, pages[b] - 1]), PAGE - tail:] = poison

    return Workload(name, B, s_q, n_heads, seq_lens, block_table, num_blocks,
                    q_nope, q_rope, w_uk, w_uv, kv_pool,
                    {"seed": seed, "pool": pool})


def preset_workload(name: str, device="cpu", **override) -> Workload:
    """Build one of ``PRESETS`` (optionally overriding B / n_heads / lens / seed)."""
    p = PRESETS[name]
    B = override.get("B", p.B)
    s_q = override.get("s_q", p.s_q)
    H = override.get("n_heads", p.n_heads)
    seed = override.get("seed", p.seed)
    lens = override.get("lens", p.lens)
    pool = override.get("pool", p.pool)
    rng = np.random.default_rng(seed + 1000)
    seq_lens = draw_seq_lens(lens, B, s_q, rng)
    w = make_workload(B, s_q, H, seq_lens, seed, pool=pool, device=device, name=name)
    w.meta["lens"] = lens
    return w


def draft_tree(B: int, s_q: int, seed: int):
    """Seeded draft trees for a speculative batch (inputs only): per sequence,
    the parent of draft i (i >= 1) is drawn uniformly from the committed
    prefix (-1) and drafts 0 .. i-1, draft 0 hangs off the prefix.  Returns
    (parents [B][s_q] int, masks int32 [B][s_q]) where bit j of masks[b][i]
    marks draft j as an ancestor of draft i or draft i itself: the visibility
    structure a drafter hands to the attention kernel."""
    rng = np.random.default_rng(seed + 2000)
    parents = [[-1] + [int(rng.integers(-1, i)) for i in range(1, s_q)] for _ in range(B)]
    masks = np.zeros((B, s_q), dtype=np.int32)
    for b, par in enumerate(parents):
        for i, pa in enumerate(par):
            masks[b, i] = (1 << i) | (masks[b, pa] if pa >= 0 else 0)
    return parents, masks
