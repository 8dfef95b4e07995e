"""Shared helpers for the GPU parity tests: run the CUDA path, run the oracle, compare."""
from __future__ import annotations

import numpy as np
import torch

from head_latent_attention_04_b200 import workloads as W
from oracle import mla_oracle as O

# Tolerances on `out` (bf16 inputs, fp32 accumulation): relative Frobenius and max abs.
REL_FRO = 5e-3
MAX_ABS = 2e-2


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def run_gpu(w: W.Workload, num_clusters=None, causal=True):
    from head_latent_attention_04_b200 import mla
    dev = torch.device("cuda")
    wd = w.to(dev)
    bt = torch.as_tensor(w.block_table, dtype=torch.int32, device=dev)
    dec = mla.Decoder(w.seq_lens, w.s_q, w.n_heads, w.max_blocks, w.num_blocks, dev,
                      causal=causal, num_clusters=num_clusters)
    res = dec.run(wd.q_nope, wd.q_rope, wd.kv_pool, bt, wd.w_uk, wd.w_uv)
    torch.cuda.synchronize()
    return dec, res


def oracle_rows(w: W.Workload, b: int, heads=None, draft_masks=None):
    """Oracle for sequence b (all its s_q rows), optionally a head subset and
    the drafts' visibility masks (one list of s_q bitmasks)."""
    rows = slice(b * w.s_q, (b + 1) * w.s_q)
    cache = w.cache_rows(b).cpu().double().numpy()
    return O.mla_decode(w.q_nope[rows].cpu().double().numpy(), w.q_rope[rows].cpu().double().numpy(),
                        [cache], w.w_uk.cpu().double().numpy(), w.w_uv.cpu().double().numpy(),
                        w.s_q, heads=heads, draft_masks=None if draft_masks is None else [draft_masks])


def oracle_all(w: W.Workload):
    out, lse, ql, ol = [], [], [], []
    for b in range(w.B):
        r = oracle_rows(w, b)
        out.append(r["out"]); lse.append(r["lse"]); ql.append(r["q_lat"]); ol.append(r["o_lat"])
    return dict(out=np.concatenate(out), lse=np.concatenate(lse), q_lat=np.concatenate(ql),
                o_lat=np.concatenate(ol))


def check_out(got, want, rel=REL_FRO, max_abs=MAX_ABS):
    g = got.float().cpu().double().numpy() if isinstance(got, torch.Tensor) else np.asarray(got)
    e = rel_fro(g, want)
    m = float(np.max(np.abs(g - want)))
    assert np.all(np.isfinite(g)), "non-finite output"
    assert e <= rel and m <= max_abs, f"rel_fro={e:.3e} (<= {rel}) max_abs={m:.3e} (<= {max_abs})"
    return e, m
