"""Host side of the C ABI (CPU only): exports, argument validation, and the split
planner checked bit-exactly against an independent Python derivation."""
import ctypes
import os
import re

import numpy as np
import pytest

from head_latent_attention_04_b200 import mla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_library_exports_every_declared_symbol():
    header = open(os.path.join(ROOT, "include", "mla.h")).read()
    declared = set(re.findall(r"^\s*(?:mla_status_t|int32_t|size_t|void|const char\*)\s+(mla_\w+)\s*\(", header, re.M))
    assert declared == set(mla.EXPORTS)
    lib = ctypes.CDLL(mla._LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    assert mla.version() >= 100


# ------------------------------------------------------------------ independent planner
ITEM_COST_PAGES = 5


def py_plan(seq_lens, s_q, causal, n_heads, num_clusters, page=64):
    """Re-derivation of the documented split rule: per query position i (its own
    group of clusters when there are at least s_q clusters), the rows are laid
    end to end in sequence order, each preceded by ITEM_COST_PAGES virtual
    pages, and the line of P' units is cut at floor(c * P' / G); a piece is a
    range's intersection with a row's real pages."""
    B = len(seq_lens)
    N = B * s_q
    rows = []
    for b in range(B):
        for i in range(s_q):
            kv = seq_lens[b] - s_q + 1 + i if causal else seq_lens[b]
            rows.append(dict(b=b, qi=i, kv=kv, pages=-(-kv // page)))
    groups = s_q if num_clusters >= s_q else 1
    G = num_clusters // groups
    pieces = []   # (cluster, row, p0, p1)
    for g in range(groups):
        members = [n for n in range(N) if groups == 1 or n % s_q == g]
        P = sum(ITEM_COST_PAGES + rows[n]["pages"] for n in members)
        off = 0
        for n in members:
            r0 = off + ITEM_COST_PAGES
            r1 = r0 + rows[n]["pages"]
            off = r1
            for c in range(G):
                lo, hi = c * P // G, (c + 1) * P // G
                a, e = max(lo, r0), min(hi, r1)
                if a < e:
                    pieces.append((g * G + c, n, a - r0, e - r0))
    count = [0] * N
    for p in pieces:
        count[p[1]] += 1
    slot_begin = [0] * (N + 1)
    for n in range(N):
        slot_begin[n + 1] = slot_begin[n] + (count[n] if count[n] > 1 else 0)
    seen = [0] * N
    items = []
    for cl, n, p0, p1 in pieces:
        k = seen[n]
        seen[n] += 1
        slot = slot_begin[n] + k if count[n] > 1 else -1
        items.append((cl, [rows[n]["b"], rows[n]["qi"], p0, p1, rows[n]["kv"], slot, n, 0]))
    items.sort(key=lambda t: t[0])          # stable: keeps row order inside a cluster
    cl_begin = [0] * (num_clusters + 1)
    for cl, _ in items:
        cl_begin[cl + 1] += 1
    for c in range(num_clusters):
        cl_begin[c + 1] += cl_begin[c]
    return cl_begin, [w for _, w in items], slot_begin


def _unpack(buf):
    off_c, off_i, off_r = buf[8], buf[9], buf[10]
    C, I, N = buf[1], buf[2], buf[4]
    return (list(buf[off_c:off_c + C + 1]),
            [list(buf[off_i + 8 * k: off_i + 8 * k + 8]) for k in range(I)],
            list(buf[off_r:off_r + N + 1]))


@pytest.mark.parametrize("case", [
    dict(lens=[4096] * 32, s_q=1, H=128, C=74),
    dict(lens=[256, 256], s_q=1, H=16, C=74),
    dict(lens=[131072] * 4, s_q=1, H=128, C=74),
    dict(lens=[1, 64, 65, 127, 128, 129, 5000], s_q=1, H=8, C=5),
    dict(lens=[2, 3, 64, 65, 66, 4097, 130], s_q=2, H=128, C=74),
    dict(lens=[2, 3, 64, 65, 66, 4097, 130], s_q=2, H=128, C=1),
    dict(lens=[77, 9000, 300], s_q=2, H=64, C=7),
    dict(lens=[3, 64, 65, 5000, 130], s_q=3, H=128, C=74),
    dict(lens=[8, 9, 700, 64], s_q=8, H=16, C=5),
    dict(lens=[4, 4100], s_q=4, H=128, C=3),
    dict(lens=[100], s_q=1, H=1, C=3),
])
def test_plan_bit_exact(case):
    dims = mla.make_dims(len(case["lens"]), case["s_q"], case["H"], max(-(-t // 64) for t in case["lens"]),
                         10 ** 6)
    buf, ns = mla.plan(dims, case["lens"], case["C"])
    assert buf[0] == 0x314C414D and buf[1] == case["C"]
    cl, items, rows = _unpack(buf)
    ecl, eitems, erows = py_plan(case["lens"], case["s_q"], True, case["H"], case["C"])
    assert cl == ecl and items == eitems and rows == erows
    assert ns == erows[-1] == buf[3]


@pytest.mark.parametrize("seed", range(6))
def test_plan_random_covers_every_page_once(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 40))
    s_q = int(rng.integers(1, 9))
    lens = rng.integers(s_q, 20000, size=B).tolist()
    C = int(rng.integers(1, 200))
    dims = mla.make_dims(B, s_q, 128, max(-(-t // 64) for t in lens), 10 ** 6)
    buf, ns = mla.plan(dims, lens, C)
    cl, items, rows = _unpack(buf)
    assert (cl, items, rows) == py_plan(lens, s_q, True, 128, C)
    covered = {}
    for w in items:
        b, qi, p0, p1, kv, slot, n = w[:7]
        assert n == b * s_q + qi and 0 <= p0 < p1 <= -(-kv // 64)
        for p in range(p0, p1):
            assert (n, p) not in covered
            covered[(n, p)] = True
    for n in range(B * s_q):
        b, qi = divmod(n, s_q)
        kv = lens[b] - s_q + 1 + qi
        assert all((n, p) in covered for p in range(-(-kv // 64)))
    pb, ob, lb = mla.plan_size(dims, C)
    assert buf[11] * 4 <= pb and ns * 128 * 512 * 4 <= ob and ns * 128 * 4 <= lb


@pytest.mark.parametrize("seed", range(4))
def test_non_causal_plan_covers_every_page_of_every_row(seed):
    # the draft-tree entry point runs non-causal plans: every query row spans its
    # sequence's whole length (the masks then pick the drafts)
    rng = np.random.default_rng(100 + seed)
    B = int(rng.integers(1, 30))
    s_q = int(rng.integers(1, 9))
    lens = rng.integers(s_q, 12000, size=B).tolist()
    C = int(rng.integers(1, 160))
    dims = mla.make_dims(B, s_q, 128, max(-(-t // 64) for t in lens), 10 ** 6, causal=False)
    buf, ns = mla.plan(dims, lens, C)
    cl, items, rows = _unpack(buf)
    assert (cl, items, rows) == py_plan(lens, s_q, False, 128, C)
    covered = set()
    for w in items:
        b, qi, p0, p1, kv, slot, n = w[:7]
        assert kv == lens[b] and n == b * s_q + qi
        covered.update((n, p) for p in range(p0, p1))
    assert covered == {(b * s_q + i, p) for b in range(B) for i in range(s_q) for p in range(-(-lens[b] // 64))}


# ------------------------------------------------------------------ validation (no GPU needed)
def test_invalid_arguments_return_codes():
    good = mla.make_dims(2, 1, 16, 4, 8)
    for field, val, code in [("d_c", 256, mla.MLA_ERR_UNSUPPORTED), ("s_q", 9, mla.MLA_ERR_UNSUPPORTED),
                             ("s_q", 0, mla.MLA_ERR_UNSUPPORTED),
                             ("n_heads", 129, mla.MLA_ERR_UNSUPPORTED), ("page_size", 32, mla.MLA_ERR_UNSUPPORTED),
                             ("B", 0, mla.MLA_ERR_INVALID_ARG), ("scale", -1.0, mla.MLA_ERR_INVALID_ARG)]:
        d = mla.make_dims(2, 1, 16, 4, 8)
        setattr(d, field, val)
        with pytest.raises(mla.MlaError) as e:
            mla.plan(d, [256, 256], 4)
        assert e.value.code == code, field
    with pytest.raises(mla.MlaError) as e:
        mla.plan(good, [256, 257], 4)                 # longer than max_blocks * 64
    assert e.value.code == mla.MLA_ERR_INVALID_ARG and "seq_lens[1]" in str(e.value)
    with pytest.raises(mla.MlaError) as e:
        mla.plan(mla.make_dims(1, 2, 16, 4, 8), [1], 4)   # T < s_q
    assert e.value.code == mla.MLA_ERR_INVALID_ARG
    # null / misaligned device pointers are rejected before any CUDA call
    lib = mla._lib
    assert lib.mla_absorb_q(None, 16, 16, 4, 16, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_absorb_q(16, 16, 16, 0, 16, None) == mla.MLA_ERR_UNSUPPORTED
    assert lib.mla_out_uv(16, 24, 16, 4, 16, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_decode_attn(ctypes.byref(good), 16, 16, 16, 16, 16, 16, 4, None, None, None, None,
                               None, None) == mla.MLA_ERR_INVALID_ARG
    assert b"o_lat" in lib.mla_last_error_string()
    assert lib.mla_combine(ctypes.byref(good), 16, None, None, 16, None, None) == mla.MLA_ERR_INVALID_ARG
    small = (ctypes.c_int32 * 4)()
    assert lib.mla_plan(ctypes.byref(good), (ctypes.c_int32 * 2)(256, 256), 4, small, 16,
                        None) == mla.MLA_ERR_WORKSPACE_TOO_SMALL


def test_plan_header_records_the_dims():
    """Header words 12 and 13 hold max_blocks_per_seq and the causal flag, which
    the kernel and the allocation-free entry point check besides B, s_q, h."""
    d = mla.make_dims(3, 2, 64, 17, 100, causal=True)
    buf, _ = mla.plan(d, [5, 700, 1000], 6)
    assert buf[5] == 64 and buf[6] == 2 and buf[7] == 3 and buf[12] == 17 and buf[13] == 1
    buf, _ = mla.plan(mla.make_dims(3, 1, 64, 17, 100, causal=False), [5, 700, 1000], 6)
    assert buf[13] == 0


def _noalloc(dims, plan, nbytes, clusters):
    """The allocation-free entry point with stand-in device pointers: every case
    below must be refused on the host, before any CUDA call."""
    return mla._lib.mla_decode_attn_combine_noalloc(ctypes.byref(dims), 16, 16, 16, 16, 16, plan.ctypes.data,
                                                    nbytes, clusters, 16, None, None, None)


def test_noalloc_refuses_plans_that_do_not_match():
    dims = mla.make_dims(4, 1, 128, 64, 1000)
    plan, _ = mla.plan(dims, [4096, 100, 3000, 64], 8)
    bad = plan.copy()
    bad[0] = 0                                                   # magic word
    assert _noalloc(dims, bad, bad.nbytes, 8) == mla.MLA_ERR_INVALID_ARG
    assert b"not a plan" in mla._lib.mla_last_error_string()
    assert _noalloc(dims, plan, plan.nbytes, 9) == mla.MLA_ERR_INVALID_ARG      # cluster count
    assert _noalloc(dims, plan, 4 * (int(plan[11]) - 1), 8) == mla.MLA_ERR_INVALID_ARG   # truncated
    assert b"plan_bytes" in mla._lib.mla_last_error_string()
    assert _noalloc(dims, plan, 60, 8) == mla.MLA_ERR_INVALID_ARG              # not even a header
    bad = plan.copy()
    bad[11] = -5                                                 # negative length
    assert _noalloc(dims, bad, bad.nbytes, 8) == mla.MLA_ERR_INVALID_ARG
    # same number of rows (B * s_q = 4), other B and s_q
    d22 = mla.make_dims(2, 2, 128, 64, 1000)
    p22, _ = mla.plan(d22, [4096, 100], 8)
    assert _noalloc(dims, p22, p22.nbytes, 8) == mla.MLA_ERR_INVALID_ARG
    assert _noalloc(d22, plan, plan.nbytes, 8) == mla.MLA_ERR_INVALID_ARG
    # a plan made for a wider block table, for the other causal flag, or for other heads
    wider, _ = mla.plan(mla.make_dims(4, 1, 128, 80, 1000), [4096, 100, 3000, 64], 8)
    assert _noalloc(dims, wider, wider.nbytes, 8) == mla.MLA_ERR_INVALID_ARG
    nc, _ = mla.plan(mla.make_dims(4, 1, 128, 64, 1000, causal=False), [4096, 100, 3000, 64], 8)
    assert _noalloc(dims, nc, nc.nbytes, 8) == mla.MLA_ERR_INVALID_ARG
    other_h, _ = mla.plan(mla.make_dims(4, 1, 64, 64, 1000), [4096, 100, 3000, 64], 8)
    assert _noalloc(dims, other_h, other_h.nbytes, 8) == mla.MLA_ERR_INVALID_ARG


def test_tree_entry_point_needs_a_non_causal_plan():
    causal = mla.make_dims(2, 4, 16, 4, 8, causal=True)
    r = mla._lib.mla_decode_attn_tree(ctypes.byref(causal), 16, 16, 16, 16, 16, 16, 16, 4, None, None, 16,
                                      None, None, None)
    assert r == mla.MLA_ERR_INVALID_ARG and b"causal" in mla._lib.mla_last_error_string()
    flat = mla.make_dims(2, 4, 16, 4, 8, causal=False)
    r = mla._lib.mla_decode_attn_tree(ctypes.byref(flat), 16, 16, 16, 16, 16, None, 16, 4, None, None, 16,
                                      None, None, None)
    assert r == mla.MLA_ERR_INVALID_ARG and b"draft_masks" in mla._lib.mla_last_error_string()


def test_fp8_entry_points_validate_before_any_launch():
    lib = mla._lib
    assert lib.mla_quantize_w_uk_fp8(16, 0, 16, 16, None) == mla.MLA_ERR_UNSUPPORTED        # n_heads
    assert lib.mla_quantize_w_uv_fp8(16, 129, 16, 16, None) == mla.MLA_ERR_UNSUPPORTED
    assert lib.mla_quantize_w_uk_fp8(None, 8, 16, 16, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_quantize_w_uv_fp8(16, 8, 16, None, None) == mla.MLA_ERR_INVALID_ARG     # scales
    assert b"w_scales" in lib.mla_last_error_string()
    assert lib.mla_quantize_rows_fp8(16, 4, 100, 16, 16, None) == mla.MLA_ERR_UNSUPPORTED   # cols % 128
    assert lib.mla_quantize_rows_fp8(16, -1, 128, 16, 16, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_quantize_rows_fp8(None, 0, 128, None, None, None) == mla.MLA_OK          # nothing to do
    assert lib.mla_quantize_rows_fp8(24, 4, 128, 16, 16, None) == mla.MLA_ERR_INVALID_ARG   # misaligned x
    assert lib.mla_absorb_q_fp8(16, 16, 16, 16, 0, 16, None) == mla.MLA_ERR_UNSUPPORTED     # n_tokens
    assert lib.mla_absorb_q_fp8(16, 16, None, 16, 4, 16, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_out_uv_fp8(16, 24, 16, 16, 4, 16, None) == mla.MLA_ERR_INVALID_ARG       # misaligned codes
    assert b"w_uv_codes" in lib.mla_last_error_string()
    assert lib.mla_out_uv_fp8(16, 16, 16, 16, 4, 200, None) == mla.MLA_ERR_UNSUPPORTED      # n_heads


def test_binding_refuses_host_and_strided_tensors():
    """A host tensor would hand a host address to a kernel, and a strided view
    would be read as if contiguous: both are refused before any CUDA call."""
    import torch
    q = torch.zeros((2, 4, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mla.absorb_q(q, torch.zeros((512, 4, 128), dtype=torch.bfloat16), torch.zeros((2, 4, 512), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="CUDA tensor"):
        mla.quantize_rows_fp8(torch.zeros((3, 128), dtype=torch.bfloat16))
    # the contiguity check, seen without a GPU through a stand-in that claims to be on one
    class FakeCuda:
        is_cuda = True
        def __init__(self, contiguous):
            self.c = contiguous
        def is_contiguous(self):
            return self.c
        def data_ptr(self):
            return 4096
    with pytest.raises(ValueError, match="contiguous"):
        mla._ptr(FakeCuda(False))
    assert mla._ptr(FakeCuda(True)) == 4096 and mla._ptr(None) is None and mla._ptr(16) == 16
