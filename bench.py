#!/usr/bin/env python
"""Benchmark of one absorbed-MLA decode step (one layer) on B200.

A step is the whole decode path on one batch: mla_absorb_q -> mla_decode_attn
-> mla_combine -> mla_out_uv, with inputs resident in HBM.  The default
workload is the largest of the decode configurations that fits one GPU, the
multi-token-prediction batch "mtp2": B=128 sequences x 2 causal query tokens,
128 heads, T lognormal (median 4096, sigma 1, capped at 32768), 64-token pages
in a random permutation of the pool, about 1 GB of latent cache.  --config
selects the others (tiny, v2_4k, varlen, long128k).  Prints ONE JSON line
(rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]
  python bench.py --path prefill|upstream|spec [...]   # the NEXT paths, one GPU, each
      kernel timed alone (spec: the mtp2 batch with --s-q draft tokens as a
      --draft chain or seeded trees)

Timing: W untimed warm-up steps; then K steps, each bracketed by its own CUDA
events on the launching stream, with L2 flushed before every step by writing
a 256 MB buffer (outside the events); the K-step region is bracketed by a
barrier and torch.cuda.synchronize() on both sides; ms_per_step is the mean
per-step event time, max over ranks.  The attention kernel alone is timed for
the roofline first in the region, as a short burst (3 replays of a CUDA graph
of 10 flush + kernel pairs, minus the flushes).  `e2e` repeats the step
through the public mla.GraphedStep API: the step's inputs (queries, page
table) copied from pinned host memory, the kernels, and the output copied back
to pinned host memory, all inside the timed region.

Multi-GPU (torchrun, one process per GPU): data-parallel replicas.  Each rank
decodes its own batch of the same shape (weak scaling); no collective runs on
the data path; timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA decode tokens/s and effective cache TB/s (% of B200 roofline)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
DECODE_SOURCES = ("head_latent_attention_04_b200/csrc/decode_attn.cu",)


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="mtp2",
                    choices=["tiny", "v2_4k", "varlen", "long128k", "mtp2"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-graph", action="store_true", help="launch the step eagerly instead of a CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--projections", default="bf16", choices=["bf16", "fp8"],
                    help="absorb / out_uv as bf16 GEMMs or as FP8 (E4M3) block-quantised BMMs")
    ap.add_argument("--cache", default="bf16", choices=["bf16", "fp8"],
                    help="latent cache rows as bf16 (1152 B/token) or E4M3 codes with fp32 block scales "
                         "and a bf16 k_rope (656 B/token)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    ap.add_argument("--path", default="decode", choices=["decode", "prefill", "upstream", "spec"],
                    help="decode: the absorbed decode step (the headline line); prefill: order-1 prefill of one "
                         "sequence (--prefill T,s); upstream: qkv_a_proj and q_up_absorb for --tokens rows")
    ap.add_argument("--prefill", default="4096,4096", help="T,s of the prefill path (s = T: full prefill)")
    ap.add_argument("--tokens", type=int, default=256, help="token rows of the upstream path")
    ap.add_argument("--s-q", type=int, default=8, help="draft tokens per sequence of the spec path (1..8)")
    ap.add_argument("--draft", default="tree", choices=["tree", "chain"],
                    help="spec path: seeded draft trees (per-query masks) or a chain (the causal rule)")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------- accounting
def algorithmic(seq_lens, s_q, H, causal=True, weight_bytes=2, cache_row_bytes=1152):
    """Algorithmic bytes / FLOPs of the step and of the attention kernel.

    Per attended (query, key) pair: 2*h*(2*d_c + d_R) FLOPs (QK over 576 +
    PV over 512 per head).  Per cached token: one cache row, read once and
    shared by all heads and all s_q query tokens of its sequence: 576 bf16 =
    1152 B, or 656 B for the FP8 cache (512 E4M3 codes, 4 fp32 scales, 64 bf16).
    ``weight_bytes``: bytes per W_UK / W_UV element (1 for E4M3 codes, whose
    scales add 4 bytes per 128 x 128 block).
    """
    T = np.asarray(seq_lens, dtype=np.int64)
    N = len(T) * s_q
    pairs = int(sum(int(t) - s_q + 1 + i if causal else int(t) for t in T for i in range(s_q)))
    cache = int(T.sum()) * cache_row_bytes
    w_bytes = 2 * 512 * H * 128 * weight_bytes + (2 * 4 * H * 4 if weight_bytes == 1 else 0)
    attn_flops = pairs * 2 * H * (2 * 512 + 64)
    bmm_flops = 2 * (2 * N * H * 128 * 512)
    q_in = N * H * (128 + 64) * 2
    out_b = N * H * 128 * 2
    attn_bytes = cache + N * H * (512 + 64) * 2 + N * H * 512 * 2
    return dict(N=N, pairs=pairs, cache_bytes=cache, step_bytes=cache + w_bytes + q_in + out_b,
                step_flops=attn_flops + bmm_flops, attn_bytes=attn_bytes, attn_flops=attn_flops)


def visible_keys(seq_lens, s_q, masks=None):
    """Keys each query row attends to, row order (b, i): the T - s_q committed
    tokens plus, for draft i, the drafts its mask marks (bit j: draft j), or
    under the causal rule drafts 0..i."""
    out = []
    for b, t in enumerate(seq_lens):
        for i in range(s_q):
            drafts = bin(int(masks[b][i]) & ((1 << s_q) - 1)).count("1") if masks is not None else i + 1
            out.append(int(t) - s_q + drafts)
    return out


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def decode_source_hash() -> str:
    h = hashlib.sha256()
    for f in DECODE_SOURCES:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(config: str):
    """DRAM bytes per attention launch from a committed ncu summary, if it still
    describes the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(p))
    except Exception:
        return None
    e = d.get(config)
    if not e or e.get("source_hash") != decode_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, uuid: str | None, index: int, period_s: float = 0.002):
        self.samples, self.reasons = [], 0
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = None
            if uuid:
                try:
                    self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
                except Exception:
                    self.h = None
            if self.h is None:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            self.reasons |= nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()
            self._sample()

    def mark(self) -> int:
        """Index of the next sample: segments of the timed region are [mark, next mark)."""
        return len(self.samples)

    def summary(self, segments=None):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        out = {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": float(self.max_mhz),
               "samples": len(self.samples), "reasons": names}
        if segments:
            seg = {}
            for name, (a, b) in segments.items():
                xs = self.samples[a:b]
                seg[name] = {"sm_mhz": float(statistics.median(xs)) if xs else None, "samples": len(xs)}
            out["segments"] = seg
        return out


# ----------------------------------------------------------------------------- CPU oracle sample
def cpu_oracle_sample(w, seconds: float, max_rows: int | None = None):
    """Times the float64 oracle on whole query rows (all heads, full context) of
    the workload until `seconds` of CPU work; returns (rows/s, rows, seconds, cores)."""
    from oracle import mla_oracle as O
    cores = len(os.sched_getaffinity(0))
    w_uk = w.w_uk.cpu().double().numpy()
    w_uv = w.w_uv.cpu().double().numpy()
    done, t0 = 0, time.perf_counter()
    order = list(range(w.B))
    for b in order:
        rows = slice(b * w.s_q, (b + 1) * w.s_q)
        cache = w.cache_rows(b).cpu().double().numpy()
        O.mla_decode(w.q_nope[rows].cpu().double().numpy(), w.q_rope[rows].cpu().double().numpy(),
                     [cache], w_uk, w_uv, w.s_q, with_intermediates=False)
        done += w.s_q
        el = time.perf_counter() - t0
        if el >= seconds or (max_rows and done >= max_rows):
            break
    el = time.perf_counter() - t0
    return done / el, done, el, cores


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_absorbed_fp32(w, b: int, w_uk=None, w_uv=None):
    """The absorbed order (order 2 of "MLA Matrix Absorption Analysis", sections
    2.2 and 3.2) for sequence b in float32 NumPy with BLAS: returns out [s][h][128]."""
    w_uk = w.w_uk.cpu().float().numpy() if w_uk is None else w_uk   # [512][h][128]
    w_uv = w.w_uv.cpu().float().numpy() if w_uv is None else w_uv
    rows = slice(b * w.s_q, (b + 1) * w.s_q)
    qn = w.q_nope[rows].cpu().float().numpy()       # [s][h][128]
    qr = w.q_rope[rows].cpu().float().numpy()       # [s][h][64]
    cache = w.cache_rows(b).cpu().float().numpy()
    ckv, kr = cache[:, :512], cache[:, 512:]
    T = cache.shape[0]
    q_lat = np.einsum("shd,khd->shk", qn, w_uk, optimize=True)
    sc = (q_lat @ ckv.T + qr @ kr.T) * np.float32(1.0 / math.sqrt(192.0))   # [s][h][T]
    for i in range(w.s_q):
        sc[i, :, T - w.s_q + 1 + i:] = -np.inf
    sc -= sc.max(-1, keepdims=True)
    p = np.exp(sc)
    p /= p.sum(-1, keepdims=True)
    return np.einsum("shk,khv->shv", p @ ckv, w_uv, optimize=True)


def cpu_absorbed_fp32_sample(w, seconds: float):
    """A fairer CPU number beside the oracle: cpu_absorbed_fp32 on whole
    sequences until `seconds`; returns (rows/s, rows, seconds)."""
    w_uk = w.w_uk.cpu().float().numpy()
    w_uv = w.w_uv.cpu().float().numpy()
    done, t0 = 0, time.perf_counter()
    for b in range(w.B):
        cpu_absorbed_fp32(w, b, w_uk, w_uv)
        done += w.s_q
        if time.perf_counter() - t0 >= seconds:
            break
    el = time.perf_counter() - t0
    return done / el, done, el


# ----------------------------------------------------------------------------- arms
def run_reference(args, rank: int, world: int):
    if rank != 0:
        return None
    from head_latent_attention_04_b200 import workloads as W
    w = W.preset_workload(args.config, device="cpu")
    rows_per_step = w.s_q                       # one sequence's query rows per step
    K, Wm = args.steps, args.warmup
    per_row_budget = None
    # warm-up on one row, then time K steps of one sequence each (cycling through the batch)
    from oracle import mla_oracle as O
    w_uk = w.w_uk.double().numpy()
    w_uv = w.w_uv.double().numpy()
    caches = {}

    def step(i):
        b = i % w.B
        rows = slice(b * w.s_q, (b + 1) * w.s_q)
        if b not in caches:
            caches[b] = w.cache_rows(b).double().numpy()
        O.mla_decode(w.q_nope[rows].double().numpy(), w.q_rope[rows].double().numpy(), [caches[b]],
                     w_uk, w_uv, w.s_q, with_intermediates=False)

    for i in range(min(Wm, 1)):
        step(i)
    t0 = time.perf_counter()
    for i in range(K):
        step(i)
    el = time.perf_counter() - t0
    value = K * rows_per_step / el
    cores = len(os.sched_getaffinity(0))
    sample = f"{K} steps x {rows_per_step} query row(s) of {args.config}, all {w.n_heads} heads, full context"
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": Wm, "ms_per_step": 1e3 * el / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args.config, w),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def workload_config(name, w):
    T = np.asarray(w.seq_lens)
    return {"workload": name, "B": int(w.B), "s_q": int(w.s_q), "n_heads": int(w.n_heads),
            "d_c": 512, "d_rope": 64, "d_nope": 128, "d_v": 128, "page_size": 64,
            "T_total": int(T.sum()), "T_min": int(T.min()), "T_max": int(T.max()),
            "pool": w.meta.get("pool"), "seed": w.meta.get("seed"),
            "l2": "flushed before every step (256 MB write, outside the step events)"}


def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    from head_latent_attention_04_b200 import dp, mla
    from head_latent_attention_04_b200 import workloads as W

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    preset = W.PRESETS[args.config]
    w = W.preset_workload(args.config, device=dev, seed=dp.replica_seed(preset.seed, rank))
    fp8 = args.projections == "fp8"
    fp8_cache = args.cache == "fp8"
    acc = algorithmic(w.seq_lens, w.s_q, w.n_heads, weight_bytes=1 if fp8 else 2,
                      cache_row_bytes=mla.FP8_ROW_BYTES if fp8_cache else 1152)
    bt = torch.as_tensor(w.block_table, device=dev)
    dec = mla.Decoder(w.seq_lens, w.s_q, w.n_heads, w.max_blocks, w.num_blocks, dev, kv_cache=args.cache)
    if fp8:   # weights quantised once, outside the timed region (static, as the weights are)
        dec.use_fp8_projections(w.w_uk, w.w_uv)
    if fp8_cache:   # the cache written once in FP8 (as a serving loop writes each new row), then resident
        pool = mla.fp8_pool_from(w.kv_pool)
        torch.cuda.synchronize()
    else:
        pool = w.kv_pool
    attn_fn = mla.decode_attn_fp8cache if fp8_cache else mla.decode_attn
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        dec.run(w.q_nope, w.q_rope, pool, bt, w.w_uk, w.w_uv)

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if dec.status.item() != 0:
        raise RuntimeError(f"device status {dec.status.item():#x} after warm-up")

    graph = None
    if not args.no_graph:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                step()
            torch.cuda.synchronize()
        except Exception as e:  # fall back to eager launches
            print(f"[bench] CUDA graph capture failed ({e}); eager launches", file=sys.stderr)
            graph = None
    run_step = graph.replay if graph is not None else step

    def barrier():
        if world > 1:
            torch.distributed.barrier(device_ids=[local_rank])
        torch.cuda.synchronize()

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    # The attention kernel alone, for the roofline: a graph of 10 (flush, attention)
    # pairs and a graph of 10 flushes are replayed in turn; the difference over 10
    # is one launch's device time (the host's launch cost stays out of it).
    attn_call = lambda: attn_fn(dec.dims, dec.q_lat, w.q_rope, pool, bt, dec.seq_lens_dev, dec.plan_dev,
                                dec.num_clusters, dec.o_part, dec.lse_part, dec.o_lat, dec.lse, dec.status)
    g_attn, g_flush = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(dev)
    with torch.cuda.stream(side):
        with torch.cuda.graph(g_attn, stream=side):
            for _ in range(10):
                flush.zero_()
                attn_call()
        with torch.cuda.graph(g_flush, stream=side):
            for _ in range(10):
                flush.zero_()
    torch.cuda.synchronize()
    # The attention kernel alone is timed as a short burst at the start of the
    # region, like the measured bf16 peak (best of 10 cuBLAS GEMMs): in a loop of
    # 200 launches on a B200 it ran into the power cap (SM clock median 1.66 GHz
    # against 1.97); the per-segment clocks in the line show what each part saw.
    R = 3
    ea = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(R)]
    ef = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(R)]
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    sampler = ClockSampler(uuid, local_rank)
    barrier()
    t_wall = time.perf_counter()
    with sampler:
        m0 = sampler.mark()
        for i in range(R):
            ea[i][0].record(stream)
            g_attn.replay()
            ea[i][1].record(stream)
            ef[i][0].record(stream)
            g_flush.replay()
            ef[i][1].record(stream)
        torch.cuda.synchronize()   # the samples after this point belong to the step loop
        m1 = sampler.mark()
        for i in range(K):
            flush.zero_()
            ev[i][0].record(stream)
            run_step()
            ev[i][1].record(stream)
        barrier()
    t_wall = time.perf_counter() - t_wall
    step_ms = [a.elapsed_time(b) for a, b in ev]
    flush_ms = statistics.fmean(a.elapsed_time(b) for a, b in ef)
    attn_ms = [(a.elapsed_time(b) - flush_ms) / 10 for a, b in ea]
    ms_local = statistics.fmean(step_ms)
    attn_local = statistics.fmean(attn_ms)
    del g_attn, g_flush
    pct = lambda xs: {"p10": float(np.percentile(xs, 10)), "p50": float(np.percentile(xs, 50)),
                      "p90": float(np.percentile(xs, 90))}
    step_pct, attn_pct = pct(step_ms), pct(attn_ms)

    # e2e, from host buffers to host buffers through the public API.
    # Serial (latency): mla.GraphedStep replays one graph per step (pinned H2D of
    # the queries and page table, the four kernels, D2H of the output), with L2
    # flushed before every step outside the events.
    gs = mla.GraphedStep(dec, pool, w.w_uk, w.w_uv)
    gs.q_nope.copy_(w.q_nope.cpu())
    gs.q_rope.copy_(w.q_rope.cpu())
    gs.block_table.copy_(torch.as_tensor(w.block_table))
    h2d, d2h = gs.h2d_bytes, gs.d2h_bytes
    for _ in range(args.warmup):
        gs.run(sync=False)
    ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    barrier()
    for i in range(K):
        flush.zero_()
        ee[i][0].record(stream)
        gs.run(sync=False)
        ee[i][1].record(stream)
    barrier()
    serial_ms = statistics.fmean(a.elapsed_time(b) for a, b in ee)
    e2e_check = bool(torch.equal(gs.out, dec.out.cpu()))
    del gs
    # Streamed (throughput): mla.StreamedDecoder overlaps each step's copies with
    # its neighbours' kernels; K back-to-back steps timed as one region.  No
    # flush inside the region: every step streams the whole KV cache, which is
    # larger than L2 for the full-size workloads.
    sd = mla.StreamedDecoder(dec, pool, w.w_uk, w.w_uv)
    for qn_h, qr_h, bt_h in sd.host_in:
        qn_h.copy_(w.q_nope.cpu())
        qr_h.copy_(w.q_rope.cpu())
        bt_h.copy_(torch.as_tensor(w.block_table))
    for _ in range(args.warmup):
        sd.submit()
    barrier()
    s_in, _, s_out = sd.streams
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for _ in range(K):
        last = sd.submit()
    e1.record(s_out)
    barrier()
    e2e_local = e0.elapsed_time(e1) / K
    e2e_check = e2e_check and bool(torch.equal(sd.wait(last), dec.out.cpu()))
    del sd
    status = int(dec.status.item())

    # bookkeeping collectives only (identity at one rank): max over ranks, status OR
    ms, attn, e2e, serial_ms = dp.reduce_max([ms_local, attn_local, e2e_local, serial_ms], device=dev)
    status = dp.reduce_status(status, device=dev)
    used_graph = graph is not None
    del graph
    if rank != 0:
        return None

    peaks, peak_src = load_peaks()
    tensor_bound = acc["attn_flops"] / (peaks["bf16_tflops"] * 1e12) > acc["attn_bytes"] / (peaks["hbm_gbs"] * 1e9)
    if tensor_bound:
        achieved = acc["attn_flops"] / (attn * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"]}
    else:
        achieved = acc["attn_bytes"] / (attn * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"]}
    roof.update({"traffic": recorded_traffic(args.config + ("_fp8cache" if fp8_cache else "")),
                 "kernel": "mla_decode_kernel" + ("<fp8 cache>" if fp8_cache else ""),
                 "alg_bytes_per_launch": acc["attn_bytes"], "alg_flops_per_launch": acc["attn_flops"],
                 "kernel_ms": attn, "peak_source": f"{peak_src} ({'MEASURED_PEAKS.json' if peak_src == 'measured' else 'recipe fallback'}, burst)"})
    step_roof_s = max(acc["step_bytes"] / (peaks["hbm_gbs"] * 1e9), acc["step_flops"] / (peaks["bf16_tflops"] * 1e12))
    tokens = acc["N"] * world
    res = {
        "metric": METRIC, "value": tokens / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": ("bf16 (attention" + ("; the latent cache stored as e4m3 codes with fp32 block scales, "
                                       "widened to bf16 on chip" if fp8_cache else "") + ")"
                  + ("; e4m3 codes with fp32 block scales (projections)" if fp8 else "")) if (fp8 or fp8_cache)
                 else "bf16",
        "data": "synthetic",
        "config": dict(workload_config(args.config, w), parallelism=f"dp{world} (independent replicas)",
                       num_clusters=dec.num_clusters, split_slots=dec.num_slots,
                       graph=used_graph, projections=args.projections, kv_cache=args.cache),
        "cache_tbs": acc["cache_bytes"] * world / (ms * 1e-3) / 1e12,
        "attn_cache_tbs": acc["cache_bytes"] / (attn * 1e-3) / 1e12,
        "tflops": acc["step_flops"] * world / (ms * 1e-3) / 1e12,
        "step_roofline_frac": step_roof_s / (ms * 1e-3),
        "ms_per_step_percentiles": step_pct,
        "attention_ms_percentiles": attn_pct,
        "attention_timing": f"{R} replays each of a CUDA graph of 10 (L2 flush, attention) pairs and of one of "
                            "10 flushes, first in the timed region (a burst, like the peak's GEMMs); per launch = "
                            "(pair graph - flush graph) / 10",
        "roofline": roof,
        "e2e": {"value": tokens / (e2e * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e,
                "path": "mla.StreamedDecoder: pinned H2D and D2H of each step overlapped with the "
                        "neighbouring steps' kernels, K steps timed as one region (KV cache > L2, no flush)",
                "serial_ms_per_step": serial_ms,
                "serial_path": "mla.GraphedStep: H2D, 4 kernels, D2H in one graph per step, L2 flushed "
                               "before each step",
                "matches_device_output": e2e_check},
        "gpu_launches": K * dec.launches_per_step + 10 * R,
        "clocks": sampler.summary({"attention": (m0, m1), "steps": (m1, None)}),
        "device_status": status,
        "wall_s_timed_region": t_wall,
    }
    if world == 1 and not args.no_cpu_baseline:
        rate, rows, secs, cores = cpu_oracle_sample(w, args.cpu_seconds)
        res["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                               "cpu_model": cpu_model(),
                               "sample": f"{rows} query rows of {args.config} (all heads, full context), "
                                         f"{secs:.1f} s, float64 order-1 oracle"}
        rate32, rows32, secs32 = cpu_absorbed_fp32_sample(w, args.cpu_seconds / 3)
        res["cpu_absorbed_fp32"] = {"value": rate32, "unit": "tokens/s", "cores": cores,
                                    "sample": f"{rows32} query rows of {args.config}, {secs32:.1f} s, "
                                              "float32 NumPy order 2 (a fairer CPU figure, not a target)"}
    return res


# ----------------------------------------------------------------------------- the NEXT paths
def _time_kernel(fn, K, W, flush, stream):
    """Device time (ms) of one fn() with L2 flushed before it: CUDA graphs of
    10 (flush, fn) pairs and of 10 flushes are replayed ceil(K / 10) times
    each, timed with CUDA events; the difference over 10 is one launch (host
    launch overhead stays out of the measurement)."""
    import torch
    for _ in range(max(W, 3)):
        flush.zero_()
        fn()
    torch.cuda.synchronize()
    g_run, g_flush = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g_run, stream=side):
            for _ in range(10):
                flush.zero_()
                fn()
        with torch.cuda.graph(g_flush, stream=side):
            for _ in range(10):
                flush.zero_()
    torch.cuda.synchronize()
    reps = max(1, (K + 9) // 10)
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    e[0].record(stream)
    for _ in range(reps):
        g_run.replay()
    e[1].record(stream)
    for _ in range(reps):
        g_flush.replay()
    e[2].record(stream)
    torch.cuda.synchronize()
    return (e[0].elapsed_time(e[1]) - e[1].elapsed_time(e[2])) / (10 * reps)


def _roof(flops, nbytes, ms, peaks, peak_src):
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    src = f"{peak_src} ({'MEASURED_PEAKS.json' if peak_src == 'measured' else 'recipe fallback'}, burst)"
    if t_tensor > t_hbm:
        a = flops / (ms * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": a, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": a / peaks["bf16_tflops"], "alg_flops": flops, "alg_bytes": nbytes, "kernel_ms": ms,
                "peak_source": src}
    a = nbytes / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": a, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": a / peaks["hbm_gbs"],
            "alg_flops": flops, "alg_bytes": nbytes, "kernel_ms": ms, "peak_source": src}


def run_next_path(args):
    """One JSON line for the prefill or upstream path (one GPU): each kernel timed
    with CUDA events on its own, L2 flushed before every run, with its roofline."""
    import torch
    from head_latent_attention_04_b200 import mla
    from head_latent_attention_04_b200 import workloads as W

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    peaks, peak_src = load_peaks()
    K, Wm = args.steps, args.warmup
    H = 128
    if args.path == "prefill":
        T, s = (int(x) for x in args.prefill.split(","))
        w = W.make_workload(1, s, H, [T], seed=7, pool="permuted", device=dev)
        row = torch.as_tensor(w.block_table[0], dtype=torch.int32, device=dev)
        k = torch.empty((T, H, 128), dtype=torch.bfloat16, device=dev)
        v = torch.empty_like(k)
        out = torch.empty((s, H, 128), dtype=torch.bfloat16, device=dev)
        up = lambda: mla.prefill_up_proj(w.kv_pool, row, T, w.w_uk, w.w_uv, k, v)
        attn = lambda: mla.prefill_attn(w.q_nope, w.q_rope, k, v, w.kv_pool, row, T, out=out)
        ms_up = _time_kernel(up, K, Wm, flush, stream)
        ms_attn = _time_kernel(attn, K, Wm, flush, stream)
        pairs = sum(T - s + 1 + i for i in range(s))
        kern = {
            "up_proj_kernel": _roof(2 * 2 * T * 512 * 128 * H, T * 1152 + 2 * 512 * H * 128 * 2 + 2 * T * H * 128 * 2,
                                    ms_up, peaks, peak_src),
            "prefill_attn_kernel": _roof(pairs * H * 2 * (192 + 128),
                                         s * H * (192 + 128) * 2 + 2 * T * H * 128 * 2 + T * 128 + s * H * 4,
                                         ms_attn, peaks, peak_src),
        }
        ms = ms_up + ms_attn
        launches = 2 * K
        tokens, workload = s, {"workload": f"prefill T={T} s={s}", "n_heads": H, "pool": "permuted", "seed": 7}
    elif args.path == "spec":
        # the mtp2 batch shape (128 sequences, lognormal lengths up to 32K) with
        # s_q draft tokens per sequence, as a chain (causal) or as seeded trees
        s_q = args.s_q
        w = W.preset_workload("mtp2", device=dev, s_q=s_q)
        tree = args.draft == "tree"
        dec = mla.Decoder(w.seq_lens, s_q, w.n_heads, w.max_blocks, w.num_blocks, dev, causal=not tree)
        bt = torch.as_tensor(w.block_table, device=dev)
        if tree:
            _, masks_np = W.draft_tree(w.B, s_q, w.meta["seed"])
            masks = torch.as_tensor(masks_np, device=dev)
        else:
            masks_np, masks = None, None
        visible = visible_keys(w.seq_lens, s_q, masks_np)
        step = lambda: dec.run(w.q_nope, w.q_rope, w.kv_pool, bt, w.w_uk, w.w_uv, draft_masks=masks)
        step()
        torch.cuda.synchronize()
        if dec.status.item() != 0:
            raise RuntimeError(f"device status {dec.status.item():#x}")
        if tree:
            attn = lambda: mla.decode_attn_tree(dec.dims, dec.q_lat, w.q_rope, w.kv_pool, bt, dec.seq_lens_dev, masks,
                                                dec.plan_dev, dec.num_clusters, dec.o_part, dec.lse_part, dec.o_lat,
                                                dec.lse, dec.status)
        else:
            attn = lambda: mla.decode_attn(dec.dims, dec.q_lat, w.q_rope, w.kv_pool, bt, dec.seq_lens_dev,
                                           dec.plan_dev, dec.num_clusters, dec.o_part, dec.lse_part, dec.o_lat,
                                           dec.lse, dec.status)
        ms_attn = _time_kernel(attn, K, Wm, flush, stream)
        ms = _time_kernel(step, K, Wm, flush, stream)
        acc = algorithmic(w.seq_lens, s_q, w.n_heads)
        flops = sum(visible) * 2 * w.n_heads * (2 * 512 + 64)
        name = "mla_decode_kernel" + ("<tree>" if tree else "")
        kern = {name: _roof(flops, acc["attn_bytes"], ms_attn, peaks, peak_src)}
        tokens = w.B * s_q
        launches = K * (1 + dec.launches_per_step)
        T = np.asarray(w.seq_lens)
        workload = {"workload": f"mtp2 batch, {s_q} draft tokens per sequence as {'seeded trees' if tree else 'a chain'}",
                    "B": int(w.B), "s_q": s_q, "n_heads": int(w.n_heads), "T_total": int(T.sum()),
                    "visible_pairs": int(sum(visible)), "seed": w.meta["seed"],
                    "step": "absorb_q + attention + combine + out_uv, one CUDA-graph replay per step"}
    else:
        N = args.tokens
        g = torch.Generator(device=dev)
        g.manual_seed(9)
        rnd = lambda shape, std: (torch.randn(shape, generator=g, device=dev) * std).to(torch.bfloat16)
        x = rnd((N, 7168), 1.0)
        w_qkv = rnd((2112, 7168), 7168 ** -0.5)
        c_q = rnd((N, 1536), 1.0)
        w_uq = rnd((1536, H, 192), 1536 ** -0.5)
        w_uk = rnd((512, H, 128), 512 ** -0.5)
        c_q_out = torch.empty((N, 1536), dtype=torch.bfloat16, device=dev)
        kv_a_out = torch.empty((N, 576), dtype=torch.bfloat16, device=dev)
        q_lat = torch.empty((N, H, 512), dtype=torch.bfloat16, device=dev)
        q_rope = torch.empty((N, H, 64), dtype=torch.bfloat16, device=dev)
        ms_a = _time_kernel(lambda: mla.qkv_a_proj(x, w_qkv, c_q_out, kv_a_out), K, Wm, flush, stream)
        ms_b = _time_kernel(lambda: mla.q_up_absorb(c_q, w_uq, w_uk, q_lat, q_rope), K, Wm, flush, stream)
        kern = {
            "qkv_a_proj_kernel": _roof(2 * N * 7168 * 2112, 2112 * 7168 * 2 + N * 7168 * 2 + N * 2112 * 2,
                                       ms_a, peaks, peak_src),
            "q_up_absorb_kernel": _roof(2 * N * 1536 * H * 192 + 2 * N * H * 128 * 512,
                                        1536 * H * 192 * 2 + 512 * H * 128 * 2 + N * 1536 * 2 + N * H * 576 * 2,
                                        ms_b, peaks, peak_src),
        }
        ms = ms_a + ms_b
        launches = 2 * K
        tokens, workload = N, {"workload": f"upstream N={N}", "n_heads": H, "seed": 9}
    return {"metric": f"{args.path} tokens/s (kernels timed one by one)", "value": tokens / (ms * 1e-3),
            "unit": "tokens/s", "n_gpus": 1, "steps": K, "warmup": Wm, "ms_per_step": ms, "higher_is_better": True,
            "dtype": "bf16", "data": "synthetic", "path": args.path,
            "config": dict(workload, l2="flushed before every kernel run (256 MB write; graphs of 10 flush + kernel "
                                        "pairs minus graphs of 10 flushes)"),
            "kernels": kern, "gpu_launches": launches}


def main(argv=None):
    args = parse_args(argv)
    if args.path != "decode":
        print(json.dumps(run_next_path(args)), flush=True)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
    else:
        import torch
        if world > 1:
            torch.cuda.set_device(local_rank)
            torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                                 device_id=torch.device("cuda", local_rank))
        try:
            res = run_ours(args, rank, world, local_rank)
        finally:
            if world > 1:
                torch.distributed.destroy_process_group()
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
