"""FP8 latent cache on the GPU against the oracle.

The cache writer (mla_kv_quantize_fp8) is compared with the oracle's
quantize_cache code by code and scale by scale (the same float32 decisions on
both sides).  The attention kernel on an FP8 pool is compared with the float64
order-1 oracle run on the dequantised cache rows (codes x scales, k_rope
unchanged); the pool it reads is written by the oracle's quantiser, never by
the CUDA path.  The kernel widens each staged row to fp16 (code x fp16(s),
relative error <= 2^-10 while the scale is an fp16 normal number), rounds
q_lat to fp16 (2^-11) and writes P as fp16 (2^-11): every operand is at least
as precise as in the bf16 kernel (2^-9), so the bf16 path's tolerances apply:
relative Frobenius <= 5e-3 and max abs <= 2e-2 on out, o_lat and q_lat, 2e-2
absolute on the LSE."""
import numpy as np
import pytest
import torch

from head_latent_attention_04_b200 import workloads as W
from oracle import fp8 as F
from oracle import mla_oracle as O
from tests.gpu_helpers import check_out

pytestmark = pytest.mark.gpu

ROW8 = 656


@pytest.fixture(scope="module")
def mla():
    from head_latent_attention_04_b200 import mla as m
    return m


def _e4m3_bytes(values: np.ndarray) -> np.ndarray:
    """E4M3 values (exactly representable) -> their code bytes."""
    return torch.from_numpy(np.ascontiguousarray(values, dtype=np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()


def oracle_pool(w: W.Workload, poison_rows=None, chunk=65536) -> torch.Tensor:
    """The FP8 pool of a workload's bf16 pool, written by the oracle quantiser:
    uint8 [num_blocks][64][656].  ``poison_rows`` (bool mask over pool rows):
    those rows get NaN codes, NaN scales and NaN k_rope instead."""
    rows = w.kv_pool.reshape(-1, 576)
    n = rows.shape[0]
    pool = np.zeros((n, ROW8), dtype=np.uint8)
    for r0 in range(0, n, chunk):
        r1 = min(n, r0 + chunk)
        codes, scales = F.quantize_cache(rows[r0:r1, :512].float().numpy())
        pool[r0:r1, :512] = _e4m3_bytes(codes)
        pool[r0:r1, 512:528] = scales.astype(np.float32).view(np.uint8).reshape(r1 - r0, 16)
        pool[r0:r1, 528:] = rows[r0:r1, 512:].contiguous().view(torch.uint8).numpy().reshape(r1 - r0, 128)
    if poison_rows is not None:
        pool[poison_rows, :512] = 0x7F                                 # E4M3 NaN
        pool[poison_rows, 512:528] = np.frombuffer(np.full(4, np.nan, np.float32).tobytes(), np.uint8)
        pool[poison_rows, 528:] = np.frombuffer(torch.full((64,), float("nan"), dtype=torch.bfloat16)
                                                .view(torch.uint8).numpy().tobytes(), np.uint8)
    return torch.from_numpy(pool.reshape(w.num_blocks, 64, ROW8))


def dequant_rows(pool_rows: np.ndarray) -> np.ndarray:
    """FP8 pool rows (uint8 [n][656]) -> float64 [n][576]: codes x scales | k_rope."""
    pool_rows = np.ascontiguousarray(pool_rows)
    out = np.empty((pool_rows.shape[0], 576), dtype=np.float64)
    scales = pool_rows[:, 512:528].copy().view(np.float32)
    out[:, :512] = F.dequantize_cache(F.e4m3_decode(pool_rows[:, :512]), scales)
    rope = torch.from_numpy(pool_rows[:, 528:].copy()).view(torch.bfloat16)
    out[:, 512:] = rope.double().numpy()
    return out


def oracle_rows8(w: W.Workload, pool8: torch.Tensor, b: int, heads=None):
    T = int(w.seq_lens[b])
    n_pages = (T + 63) // 64
    ids = np.asarray(w.block_table[b, :n_pages], dtype=np.int64)
    cache = dequant_rows(pool8.numpy()[ids].reshape(-1, ROW8)[:T])
    rows = slice(b * w.s_q, (b + 1) * w.s_q)
    return O.mla_decode(w.q_nope[rows].double().numpy(), w.q_rope[rows].double().numpy(), [cache],
                        w.w_uk.double().numpy(), w.w_uv.double().numpy(), w.s_q, heads=heads)


def run_fp8(mla, w: W.Workload, pool8: torch.Tensor, num_clusters=None):
    dev = torch.device("cuda")
    wd = w.to(dev)
    bt = torch.as_tensor(w.block_table, dtype=torch.int32, device=dev)
    dec = mla.Decoder(w.seq_lens, w.s_q, w.n_heads, w.max_blocks, w.num_blocks, dev,
                      num_clusters=num_clusters, kv_cache="fp8")
    res = dec.run(wd.q_nope, wd.q_rope, pool8.to(dev), bt, wd.w_uk, wd.w_uv)
    torch.cuda.synchronize()
    return dec, res


def full_check8(mla, w, num_clusters=None, poison_rows=None):
    pool8 = oracle_pool(w, poison_rows)
    dec, res = run_fp8(mla, w, pool8, num_clusters)
    assert res.status.item() == 0
    for b in range(w.B):
        ref = oracle_rows8(w, pool8, b)
        rows = slice(b * w.s_q, (b + 1) * w.s_q)
        check_out(res.out[rows], ref["out"])
        check_out(res.o_lat[rows], ref["o_lat"])
        check_out(res.q_lat[rows], ref["q_lat"])
        np.testing.assert_allclose(res.lse[rows].cpu().numpy(), ref["lse"], rtol=0, atol=2e-2)
    return dec, res


# ------------------------------------------------------------------ the cache writer
def test_kv_quantize_is_bit_exact(mla):
    gen = torch.Generator().manual_seed(7)
    n, nb = 333, 8
    kv = torch.randn((n, 576), generator=gen).to(torch.bfloat16)
    kv[5, 256:384] = 0                      # an all-zero block takes scale 1
    kv[7, :128] *= 1000                     # blocks of very different ranges
    kv[9, 384:512] *= 1e-3
    slots = torch.from_numpy(np.random.default_rng(3).permutation(nb * 64)[:n].astype(np.int32))
    dev = torch.device("cuda")
    pool = torch.full((nb, 64, ROW8), 0xAB, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    mla.kv_quantize_fp8(kv.to(dev), slots.to(dev), pool, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    got = pool.reshape(-1, ROW8).cpu().numpy()
    codes, scales = F.quantize_cache(kv[:, :512].float().numpy())
    s = slots.numpy()
    assert np.array_equal(F.e4m3_decode(got[s, :512]), codes)
    assert np.array_equal(got[s, 512:528].copy().view(np.float32), scales.astype(np.float32))
    assert np.array_equal(got[s, 528:], kv[:, 512:].contiguous().view(torch.uint8).numpy().reshape(n, 128))
    untouched = np.setdiff1d(np.arange(nb * 64), s)
    assert np.all(got[untouched] == 0xAB)


def test_kv_quantize_flags_blocks_beyond_fp16(mla):
    """A block with amax > 65504 is written (bit-exact as ever) and flagged:
    the attention kernel widens rows to fp16."""
    dev = torch.device("cuda")
    kv = torch.randn((4, 576), generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    kv[2, 128:256] *= 1e5
    pool = torch.zeros((1, 64, ROW8), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    mla.kv_quantize_fp8(kv.to(dev), torch.arange(4, dtype=torch.int32, device=dev), pool, status)
    torch.cuda.synchronize()
    assert status.item() == mla.STATUS_CACHE_RANGE
    got = pool.reshape(-1, ROW8)[:4].cpu().numpy()
    codes, scales = F.quantize_cache(kv[:, :512].float().numpy())
    assert np.array_equal(F.e4m3_decode(got[:, :512]), codes)
    assert np.array_equal(got[:, 512:528].copy().view(np.float32), scales.astype(np.float32))


def test_kv_quantize_bad_slot_reports_and_skips(mla):
    dev = torch.device("cuda")
    kv = torch.randn((3, 576), generator=torch.Generator().manual_seed(1)).to(torch.bfloat16).to(dev)
    pool = torch.full((2, 64, ROW8), 0x11, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    slots = torch.tensor([-1, 5, 128], dtype=torch.int32, device=dev)
    mla.kv_quantize_fp8(kv, slots, pool, status)
    torch.cuda.synchronize()
    assert status.item() == mla.STATUS_BAD_BLOCK
    p = pool.reshape(-1, ROW8).cpu().numpy()
    assert np.all(np.delete(p, 5, axis=0) == 0x11)
    assert not np.all(p[5] == 0x11)


# ------------------------------------------------------------------ attention on the FP8 pool
def test_fp8cache_tiny(mla):
    full_check8(mla, W.preset_workload("tiny"))


@pytest.mark.parametrize("clusters", [1, 3, 74, 148])
def test_fp8cache_split_counts(mla, clusters):
    w = W.make_workload(3, 1, 32, [700, 64, 1000], seed=11, pool="permuted")
    full_check8(mla, w, num_clusters=clusters)


@pytest.mark.parametrize("lens", [[1], [65], [1, 2, 3, 127, 128, 129, 191]])
def test_fp8cache_ragged_lengths(mla, lens):
    w = W.make_workload(len(lens), 1, 128, lens, seed=sum(lens) + 1, pool="scattered:1.5")
    full_check8(mla, w, num_clusters=4)


@pytest.mark.parametrize("H", [1, 100])
def test_fp8cache_head_counts(mla, H):
    w = W.make_workload(2, 1, H, [300, 90], seed=H + 2, pool="permuted")
    full_check8(mla, w)


@pytest.mark.parametrize("s_q,lens,clusters", [(2, [2, 3, 65, 66, 200], 74), (4, [4, 200, 4100], 7)])
def test_fp8cache_speculative_causal(mla, s_q, lens, clusters):
    w = W.make_workload(len(lens), s_q, 128, lens, seed=s_q * 5 + clusters, pool="permuted")
    full_check8(mla, w, num_clusters=clusters)


@pytest.mark.parametrize("s_q,lens,clusters", [(1, [65, 130, 1, 200, 64], 5), (2, [66, 129, 2], 74)])
def test_fp8cache_non_finite_rows_never_leak(mla, s_q, lens, clusters):
    """Page tails and unused pool blocks hold NaN codes, NaN scales and NaN
    k_rope: they are never widened into the product (zero-filled shifted
    loads), so the output stays finite and matches."""
    w = W.make_workload(len(lens), s_q, 128, lens, seed=91 + s_q, pool="scattered:3")
    used = np.zeros((w.num_blocks, 64), dtype=bool)
    for b in range(w.B):
        T = int(w.seq_lens[b])
        for p in range((T + 63) // 64):
            used[int(w.block_table[b, p]), :min(64, T - 64 * p)] = True
    full_check8(mla, w, num_clusters=clusters, poison_rows=~used.reshape(-1))


def test_fp8cache_matches_bf16_kernel_on_exact_rows(mla):
    """Cache values that are exact E4M3 codes times power-of-two scales are
    bf16 values, so the FP8 pool and the bf16 pool hold the same numbers (the
    oracle's dequantised rows equal the bf16 rows exactly): the two kernels
    then agree with the oracle and with each other (they differ only in the
    fp16 / bf16 rounding of q_lat and P)."""
    w = W.make_workload(3, 2, 128, [300, 1000, 70], seed=13, pool="permuted")
    g = torch.Generator().manual_seed(5)
    lat = torch.randint(-448, 449, (w.num_blocks, 64, 512), generator=g).float()
    lat = torch.from_numpy(F.e4m3_round(lat.numpy()).astype(np.float32))
    exps = (-9, -10, -11, -8)                   # per block: amax 448 -> scale amax / 448, a power of two,
    for j, e in enumerate(exps):                # and values of order one (the unit-variance workloads' size)
        lat[..., 128 * j:128 * (j + 1)] *= 2.0 ** e
        lat[..., 128 * j] = 448 * 2.0 ** e      # every block of every row reaches its amax
    w.kv_pool[..., :512] = lat.to(torch.bfloat16)
    assert torch.equal(w.kv_pool[..., :512].float(), lat)
    pool8 = oracle_pool(w)
    assert np.array_equal(dequant_rows(pool8.numpy().reshape(-1, ROW8))[:, :512], lat.reshape(-1, 512).double().numpy())
    _, r8 = run_fp8(mla, w, pool8, num_clusters=9)
    from tests.gpu_helpers import run_gpu, rel_fro
    _, r16 = run_gpu(w, num_clusters=9)
    assert r8.status.item() == 0 and r16.status.item() == 0
    for b in range(w.B):
        ref = oracle_rows8(w, pool8, b)
        rows = slice(b * w.s_q, (b + 1) * w.s_q)
        check_out(r8.o_lat[rows], ref["o_lat"])
        check_out(r16.o_lat[rows], ref["o_lat"])
        check_out(r8.out[rows], ref["out"])
    assert rel_fro(r8.o_lat.float().cpu().numpy(), r16.o_lat.float().cpu().numpy()) < 5e-3


# ------------------------------------------------------------------ full-size, sampled
@pytest.mark.parametrize("name,heads", [("v2_4k", None), ("long128k", list(range(5, 128, 8)))])
def test_fp8cache_full_size(mla, name, heads):
    """A full-size preset on the FP8 pool (the bench's launch configuration):
    every head of one split sequence (v2_4k), or 16 heads over all four TMEM
    lane quarters of one 128K-token sequence."""
    w = W.preset_workload(name)
    pool8 = oracle_pool(w)
    dec, res = run_fp8(mla, w, pool8)
    assert res.status.item() == 0 and dec.num_slots > 0
    out = res.out.float().cpu().numpy()
    assert np.all(np.isfinite(out))
    rs = dec.plan_host[dec.plan_host[10]:dec.plan_host[10] + w.N + 1]
    b = max(range(w.B), key=lambda i: (int(rs[i + 1] - rs[i]), -i))
    ref = oracle_rows8(w, pool8, b, heads=heads)
    rows = slice(b * w.s_q, (b + 1) * w.s_q)
    got = res.out[rows] if heads is None else res.out[rows][:, heads]
    check_out(got, ref["out"])
    got_ol = res.o_lat[rows] if heads is None else res.o_lat[rows][:, heads]
    check_out(got_ol, ref["o_lat"])


@pytest.mark.parametrize("s_q,H,lens,clusters", [(8, 128, [8, 9, 70, 640], 74), (3, 33, [3, 64, 200, 1000], 6)])
def test_fp8cache_long_speculation_and_odd_heads(mla, s_q, H, lens, clusters):
    """s_q up to 8 causal drafts, and a head count that ends inside a TMEM lane quarter."""
    w = W.make_workload(len(lens), s_q, H, lens, seed=101 + s_q + H, pool="scattered:2")
    full_check8(mla, w, num_clusters=clusters)


def test_fp8cache_stale_lengths_are_rejected(mla):
    """The FP8 instance checks the device seq_lens against the plan like the bf16 one."""
    w = W.make_workload(3, 1, 128, [300, 1000, 77], seed=57, pool="scattered:2")
    pool8 = oracle_pool(w)
    dev = torch.device("cuda")
    dec, res = run_fp8(mla, w, pool8, num_clusters=4)
    assert res.status.item() == 0
    dec.seq_lens_dev[1] += 1
    dec.status.zero_()
    wd = w.to(dev)
    r = dec.run(wd.q_nope, wd.q_rope, pool8.to(dev), torch.as_tensor(w.block_table, device=dev), wd.w_uk, wd.w_uv)
    torch.cuda.synchronize()
    assert r.status.item() == mla.STATUS_BAD_SEQLEN
    assert torch.all(r.out[1] == 0) and torch.all(torch.isneginf(r.lse[1]))
    for b in (0, 2):
        check_out(r.out[b:b + 1], oracle_rows8(w, pool8, b)["out"])


def test_fp8cache_wait_time_out_returns_and_recovers(mla):
    """Bounded waits in the FP8 instance (the widening waits included): with a
    1 ns bound the kernel gives up with MLA_STATUS_TIMEOUT and returns, and the
    next call with the default bound matches the oracle."""
    w = W.make_workload(3, 2, 128, [2000, 70, 600], seed=68, pool="permuted")
    pool8 = oracle_pool(w)
    try:
        mla.set_wait_limit_ns(1)
        for _ in range(2):
            _, res = run_fp8(mla, w, pool8, num_clusters=6)
            assert res.status.item() & mla.STATUS_TIMEOUT
    finally:
        mla.set_wait_limit_ns(0)
    _, res = run_fp8(mla, w, pool8, num_clusters=6)
    assert res.status.item() == 0
    for b in range(w.B):
        check_out(res.out[b * 2:(b + 1) * 2], oracle_rows8(w, pool8, b)["out"])
