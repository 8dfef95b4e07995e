"""ctypes binding of libmla (include/mla.h): argument marshalling only.

Every step of the decode path runs in the library's CUDA kernels; this module
turns torch tensors into device pointers and the current CUDA stream into a
cudaStream_t, and raises on error codes.  Importing it fails loudly when the
shared library has not been built: there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import numpy as np
import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libmla.so is not built ({_LIB_PATH}); run "
                      "`python -m head_latent_attention_04_b200.build`")
_lib = ctypes.CDLL(_LIB_PATH)

MLA_OK, MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED = 0, 1, 2
MLA_ERR_WORKSPACE_TOO_SMALL, MLA_ERR_CUDA, MLA_ERR_TIMEOUT = 3, 4, 5
STATUS_BAD_BLOCK, STATUS_TIMEOUT, STATUS_BAD_SEQLEN, STATUS_BAD_PLAN, STATUS_SCORE_RANGE = 0x1, 0x2, 0x4, 0x8, 0x10
STATUS_CACHE_RANGE = 0x20
EXPORTS = ("mla_version", "mla_last_error_string", "mla_absorb_q", "mla_out_uv",
           "mla_max_clusters", "mla_plan_size", "mla_plan", "mla_decode_attn", "mla_combine",
           "mla_debug_gather_pages", "mla_decode_attn_combine_noalloc", "mla_noalloc_scratch_bytes",
           "mla_quantize_w_uk_fp8", "mla_quantize_w_uv_fp8", "mla_quantize_rows_fp8", "mla_absorb_q_fp8",
           "mla_out_uv_fp8", "mla_set_wait_limit_ns", "mla_decode_attn_tree", "mla_prefill_up_proj",
           "mla_prefill_attn", "mla_qkv_a_proj", "mla_q_up_absorb", "mla_decode_attn_fp8cache",
           "mla_kv_quantize_fp8")


class MlaDims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("s_q", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("d_nope", ctypes.c_int32), ("d_rope", ctypes.c_int32), ("d_c", ctypes.c_int32),
                ("d_v", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("max_blocks_per_seq", ctypes.c_int32), ("num_blocks", ctypes.c_int32),
                ("scale", ctypes.c_float), ("causal", ctypes.c_int32)]


_vp, _i32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
_pdims = ctypes.POINTER(MlaDims)
_lib.mla_version.restype = _i32
_lib.mla_last_error_string.restype = ctypes.c_char_p
for _name, _args in {
    "mla_absorb_q": [_vp, _vp, _vp, _i32, _i32, _vp],
    "mla_out_uv": [_vp, _vp, _vp, _i32, _i32, _vp],
    "mla_max_clusters": [ctypes.POINTER(_i32)],
    "mla_plan_size": [_pdims, _i32, ctypes.POINTER(_sz), ctypes.POINTER(_sz), ctypes.POINTER(_sz)],
    "mla_plan": [_pdims, _vp, _i32, _vp, _sz, ctypes.POINTER(_i32)],
    "mla_decode_attn": [_pdims, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp],
    "mla_decode_attn_tree": [_pdims, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp],
    "mla_decode_attn_fp8cache": [_pdims, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp],
    "mla_kv_quantize_fp8": [_vp, _vp, ctypes.c_int64, _vp, _i32, _vp, _vp],
    "mla_combine": [_pdims, _vp, _vp, _vp, _vp, _vp, _vp],
    "mla_debug_gather_pages": [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp],
    "mla_decode_attn_combine_noalloc": [_pdims, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _i32, _vp, _vp, _vp, _vp],
    "mla_quantize_w_uk_fp8": [_vp, _i32, _vp, _vp, _vp],
    "mla_quantize_w_uv_fp8": [_vp, _i32, _vp, _vp, _vp],
    "mla_quantize_rows_fp8": [_vp, ctypes.c_int64, _i32, _vp, _vp, _vp],
    "mla_absorb_q_fp8": [_vp, _vp, _vp, _vp, _i32, _i32, _vp],
    "mla_out_uv_fp8": [_vp, _vp, _vp, _vp, _i32, _i32, _vp],
    "mla_prefill_up_proj": [_vp, _vp, _i32, _i32, _vp, _vp, _i32, _vp, _vp, _vp],
    "mla_qkv_a_proj": [_vp, _vp, _vp, _vp, _i32, _vp],
    "mla_q_up_absorb": [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _vp],
    "mla_prefill_attn": [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, ctypes.c_float, _vp, _vp, _vp],
}.items():
    getattr(_lib, _name).argtypes = _args
    getattr(_lib, _name).restype = _i32


_lib.mla_noalloc_scratch_bytes.argtypes = []
_lib.mla_noalloc_scratch_bytes.restype = _sz
_lib.mla_set_wait_limit_ns.argtypes = [ctypes.c_int64]
_lib.mla_set_wait_limit_ns.restype = None


class MlaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = _lib.mla_last_error_string().decode(errors="replace")
        super().__init__(f"{where}: status {code}: {msg}")


def _check(code: int, where: str):
    if code != MLA_OK:
        raise MlaError(code, where)


def _ptr(t) -> int | None:
    """Device address of a tensor argument.  The library reads raw pointers,
    so a host tensor (a host address handed to a kernel) or a strided view
    (read as if contiguous) is refused here, before anything is launched."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError(f"expected a CUDA tensor, got one on {t.device}")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor (the library assumes row-major layouts)")
    return t.data_ptr()


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def version() -> int:
    return _lib.mla_version()


def make_dims(B, s_q, n_heads, max_blocks, num_blocks, scale=None, causal=True) -> MlaDims:
    if scale is None:
        scale = 1.0 / math.sqrt(128 + 64)
    return MlaDims(B, s_q, n_heads, 128, 64, 512, 128, 64, max_blocks, num_blocks, float(scale),
                   1 if causal else 0)


def set_wait_limit_ns(ns: int) -> None:
    """Bound on each pipeline wait of decode launches made from now on
    (process-wide; 0 restores the 200 ms default).  A wait past it makes the
    kernel give up cleanly with STATUS_TIMEOUT."""
    _lib.mla_set_wait_limit_ns(int(ns))


def max_clusters() -> int:
    n = _i32(0)
    _check(_lib.mla_max_clusters(ctypes.byref(n)), "mla_max_clusters")
    return n.value


def plan_size(dims: MlaDims, num_clusters: int):
    pb, ob, lb = _sz(0), _sz(0), _sz(0)
    _check(_lib.mla_plan_size(ctypes.byref(dims), num_clusters, ctypes.byref(pb), ctypes.byref(ob),
                              ctypes.byref(lb)), "mla_plan_size")
    return pb.value, ob.value, lb.value


def plan(dims: MlaDims, seq_lens, num_clusters: int):
    """Host plan as an int32 numpy array, and the number of partial slots used."""
    pb, _, _ = plan_size(dims, num_clusters)
    buf = np.zeros(pb // 4, dtype=np.int32)
    sl = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    ns = _i32(0)
    _check(_lib.mla_plan(ctypes.byref(dims), sl.ctypes.data, num_clusters, buf.ctypes.data, pb,
                         ctypes.byref(ns)), "mla_plan")
    return buf, ns.value


def absorb_q(q_nope: torch.Tensor, w_uk: torch.Tensor, out: torch.Tensor | None = None, stream=None):
    N, H, _ = q_nope.shape
    if out is None:
        out = torch.empty((N, H, 512), dtype=torch.bfloat16, device=q_nope.device)
    _check(_lib.mla_absorb_q(_ptr(q_nope), _ptr(w_uk), _ptr(out), N, H, _stream(stream)), "mla_absorb_q")
    return out


def out_uv(o_lat: torch.Tensor, w_uv: torch.Tensor, out: torch.Tensor | None = None, stream=None):
    N, H, _ = o_lat.shape
    if out is None:
        out = torch.empty((N, H, 128), dtype=torch.bfloat16, device=o_lat.device)
    _check(_lib.mla_out_uv(_ptr(o_lat), _ptr(w_uv), _ptr(out), N, H, _stream(stream)), "mla_out_uv")
    return out


@dataclass
class Fp8Weight:
    """A projection weight as E4M3 codes (uint8) and fp32 block scales [H][4]."""
    codes: torch.Tensor
    scales: torch.Tensor


def quantize_w_uk_fp8(w_uk: torch.Tensor, stream=None) -> Fp8Weight:
    """W_UK bf16 [512][H][128] -> codes [H][512][128] and scales [H][4]."""
    H = w_uk.shape[1]
    codes = torch.empty((H, 512, 128), dtype=torch.uint8, device=w_uk.device)
    scales = torch.empty((H, 4), dtype=torch.float32, device=w_uk.device)
    _check(_lib.mla_quantize_w_uk_fp8(_ptr(w_uk), H, _ptr(codes), _ptr(scales), _stream(stream)),
           "mla_quantize_w_uk_fp8")
    return Fp8Weight(codes, scales)


def quantize_w_uv_fp8(w_uv: torch.Tensor, stream=None) -> Fp8Weight:
    """W_UV bf16 [512][H][128] -> codes [H][128][512] and scales [H][4]."""
    H = w_uv.shape[1]
    codes = torch.empty((H, 128, 512), dtype=torch.uint8, device=w_uv.device)
    scales = torch.empty((H, 4), dtype=torch.float32, device=w_uv.device)
    _check(_lib.mla_quantize_w_uv_fp8(_ptr(w_uv), H, _ptr(codes), _ptr(scales), _stream(stream)),
           "mla_quantize_w_uv_fp8")
    return Fp8Weight(codes, scales)


def quantize_rows_fp8(x: torch.Tensor, stream=None):
    """bf16 [..., cols] -> (codes uint8 [..., cols], scales fp32 [..., cols / 128])."""
    cols = x.shape[-1]
    rows = x.numel() // cols
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    scales = torch.empty(tuple(x.shape[:-1]) + (cols // 128,), dtype=torch.float32, device=x.device)
    _check(_lib.mla_quantize_rows_fp8(_ptr(x), rows, cols, _ptr(codes), _ptr(scales), _stream(stream)),
           "mla_quantize_rows_fp8")
    return codes, scales


def absorb_q_fp8(q_nope: torch.Tensor, w: Fp8Weight, out: torch.Tensor | None = None, stream=None):
    N, H, _ = q_nope.shape
    if out is None:
        out = torch.empty((N, H, 512), dtype=torch.bfloat16, device=q_nope.device)
    _check(_lib.mla_absorb_q_fp8(_ptr(q_nope), _ptr(w.codes), _ptr(w.scales), _ptr(out), N, H, _stream(stream)),
           "mla_absorb_q_fp8")
    return out


def out_uv_fp8(o_lat: torch.Tensor, w: Fp8Weight, out: torch.Tensor | None = None, stream=None):
    N, H, _ = o_lat.shape
    if out is None:
        out = torch.empty((N, H, 128), dtype=torch.bfloat16, device=o_lat.device)
    _check(_lib.mla_out_uv_fp8(_ptr(o_lat), _ptr(w.codes), _ptr(w.scales), _ptr(out), N, H, _stream(stream)),
           "mla_out_uv_fp8")
    return out


def decode_attn(dims, q_lat, q_rope, kv_pool, block_table, seq_lens, plan_dev, num_clusters,
                o_part, lse_part, o_lat, lse_out=None, status=None, stream=None):
    _check(_lib.mla_decode_attn(ctypes.byref(dims), _ptr(q_lat), _ptr(q_rope), _ptr(kv_pool),
                                _ptr(block_table), _ptr(seq_lens), _ptr(plan_dev), num_clusters,
                                _ptr(o_part), _ptr(lse_part), _ptr(o_lat), _ptr(lse_out),
                                _ptr(status), _stream(stream)), "mla_decode_attn")


def decode_attn_tree(dims, q_lat, q_rope, kv_pool, block_table, seq_lens, draft_masks, plan_dev, num_clusters,
                     o_part, lse_part, o_lat, lse_out=None, status=None, stream=None):
    """decode_attn for drafts that form a tree: ``draft_masks`` int32 [B][s_q]
    (device), bit j of row i = draft j visible to query i (dims.causal must be 0)."""
    _check(_lib.mla_decode_attn_tree(ctypes.byref(dims), _ptr(q_lat), _ptr(q_rope), _ptr(kv_pool),
                                     _ptr(block_table), _ptr(seq_lens), _ptr(draft_masks), _ptr(plan_dev),
                                     num_clusters, _ptr(o_part), _ptr(lse_part), _ptr(o_lat), _ptr(lse_out),
                                     _ptr(status), _stream(stream)), "mla_decode_attn_tree")


FP8_ROW_BYTES = 656   # 512 E4M3 codes | 4 fp32 block scales | 64 bf16 k_rope


def decode_attn_fp8cache(dims, q_lat, q_rope, kv_pool_fp8, block_table, seq_lens, plan_dev, num_clusters,
                         o_part, lse_part, o_lat, lse_out=None, status=None, stream=None):
    """decode_attn on an FP8 latent cache: ``kv_pool_fp8`` uint8
    [num_blocks][64][656] as :func:`kv_quantize_fp8` writes it."""
    _check(_lib.mla_decode_attn_fp8cache(ctypes.byref(dims), _ptr(q_lat), _ptr(q_rope), _ptr(kv_pool_fp8),
                                         _ptr(block_table), _ptr(seq_lens), _ptr(plan_dev), num_clusters,
                                         _ptr(o_part), _ptr(lse_part), _ptr(o_lat), _ptr(lse_out),
                                         _ptr(status), _stream(stream)), "mla_decode_attn_fp8cache")


def kv_quantize_fp8(kv, slots, kv_pool_fp8, status=None, stream=None):
    """bf16 cache rows ``kv`` [n][576] -> slots ``slots`` (int32 [n], block * 64 +
    row) of the FP8 pool (uint8 [num_blocks][64][656])."""
    n = kv.numel() // 576
    _check(_lib.mla_kv_quantize_fp8(_ptr(kv), _ptr(slots), n, _ptr(kv_pool_fp8), kv_pool_fp8.shape[0],
                                    _ptr(status), _stream(stream)), "mla_kv_quantize_fp8")
    return kv_pool_fp8


def fp8_pool_from(kv_pool, stream=None):
    """The FP8 copy of a whole bf16 pool [num_blocks][64][576] (every slot quantised)."""
    nb = kv_pool.shape[0]
    pool8 = torch.empty((nb, 64, FP8_ROW_BYTES), dtype=torch.uint8, device=kv_pool.device)
    slots = torch.arange(nb * 64, dtype=torch.int32, device=kv_pool.device)
    return kv_quantize_fp8(kv_pool.reshape(nb * 64, 576), slots, pool8, stream=stream)


def combine(dims, plan_dev, o_part, lse_part, o_lat, lse_out=None, stream=None):
    _check(_lib.mla_combine(ctypes.byref(dims), _ptr(plan_dev), _ptr(o_part), _ptr(lse_part),
                            _ptr(o_lat), _ptr(lse_out), _stream(stream)), "mla_combine")


def qkv_a_proj(x, w_qkv_a, c_q=None, kv_a=None, stream=None):
    """Fused down-projections: x [N][7168] -> c_q [N][1536], kv_a [N][576]."""
    N = x.shape[0]
    if c_q is None:
        c_q = torch.empty((N, 1536), dtype=torch.bfloat16, device=x.device)
    if kv_a is None:
        kv_a = torch.empty((N, 576), dtype=torch.bfloat16, device=x.device)
    _check(_lib.mla_qkv_a_proj(_ptr(x), _ptr(w_qkv_a), _ptr(c_q), _ptr(kv_a), N, _stream(stream)), "mla_qkv_a_proj")
    return c_q, kv_a


def q_up_absorb(c_q, w_uq, w_uk, q_lat=None, q_rope=None, stream=None):
    """c_q [N][1536] -> q_lat [N][h][512] (through W_UQ then W_UK) and q_rope [N][h][64]."""
    N, H = c_q.shape[0], w_uq.shape[1]
    if q_lat is None:
        q_lat = torch.empty((N, H, 512), dtype=torch.bfloat16, device=c_q.device)
    if q_rope is None:
        q_rope = torch.empty((N, H, 64), dtype=torch.bfloat16, device=c_q.device)
    _check(_lib.mla_q_up_absorb(_ptr(c_q), _ptr(w_uq), _ptr(w_uk), _ptr(q_lat), _ptr(q_rope), N, H, _stream(stream)),
           "mla_q_up_absorb")
    return q_lat, q_rope


def prefill_up_proj(kv_pool, block_row, T, w_uk, w_uv, k_out=None, v_out=None, stream=None):
    """K and V [T][h][128] of one sequence's first T cached tokens (order 1)."""
    H = w_uk.shape[1]
    if k_out is None:
        k_out = torch.empty((T, H, 128), dtype=torch.bfloat16, device=kv_pool.device)
    if v_out is None:
        v_out = torch.empty((T, H, 128), dtype=torch.bfloat16, device=kv_pool.device)
    _check(_lib.mla_prefill_up_proj(_ptr(kv_pool), _ptr(block_row), T, kv_pool.shape[0], _ptr(w_uk), _ptr(w_uv), H,
                                    _ptr(k_out), _ptr(v_out), _stream(stream)), "mla_prefill_up_proj")
    return k_out, v_out


def prefill_attn(q_nope, q_rope, k, v, kv_pool, block_row, T, scale=None, out=None, lse=None, stream=None):
    """Causal attention of the last s = q_nope.shape[0] of T cached tokens."""
    s, H, _ = q_nope.shape
    if scale is None:
        scale = 1.0 / math.sqrt(128 + 64)
    if out is None:
        out = torch.empty((s, H, 128), dtype=torch.bfloat16, device=q_nope.device)
    _check(_lib.mla_prefill_attn(_ptr(q_nope), _ptr(q_rope), _ptr(k), _ptr(v), _ptr(kv_pool), _ptr(block_row), T, s,
                                 H, kv_pool.shape[0], float(scale), _ptr(out), _ptr(lse), _stream(stream)),
           "mla_prefill_attn")
    return out


def prefill(q_nope, q_rope, kv_pool, block_row, T, w_uk, w_uv, scale=None, lse=None, stream=None):
    """Prefill (s = T) or a prefill chunk (s < T) of one sequence in order 1."""
    k, v = prefill_up_proj(kv_pool, block_row, T, w_uk, w_uv, stream=stream)
    return prefill_attn(q_nope, q_rope, k, v, kv_pool, block_row, T, scale=scale, lse=lse, stream=stream)


def noalloc_scratch_bytes() -> int:
    """Size of the library-owned device array used by ``decode_attn_combine_noalloc``."""
    return _lib.mla_noalloc_scratch_bytes()


def decode_attn_combine_noalloc(dims, q_lat, q_rope, kv_pool, block_table, seq_lens, plan_host: np.ndarray,
                                num_clusters, o_lat, lse_out=None, status=None, stream=None):
    """Attention + split merge with no caller workspace and no device allocation.

    For callers that may not allocate device memory (e.g. a runtime that has
    pre-reserved HBM for its KV cache): ``plan_host`` is the host plan from
    :func:`plan`; the plan copy and the partial outputs live in a fixed array
    inside the library (see :func:`noalloc_scratch_bytes`).
    """
    pl = np.ascontiguousarray(plan_host, dtype=np.int32)
    _check(_lib.mla_decode_attn_combine_noalloc(ctypes.byref(dims), _ptr(q_lat), _ptr(q_rope), _ptr(kv_pool),
                                                _ptr(block_table), _ptr(seq_lens), pl.ctypes.data, pl.nbytes,
                                                num_clusters, _ptr(o_lat), _ptr(lse_out), _ptr(status),
                                                _stream(stream)), "mla_decode_attn_combine_noalloc")


def debug_gather_pages(kv_pool, block_table, b, n_pages, max_blocks, num_blocks, out, status=None,
                       stream=None):
    _check(_lib.mla_debug_gather_pages(_ptr(kv_pool), _ptr(block_table), b, n_pages, max_blocks,
                                       num_blocks, _ptr(out), _ptr(status), _stream(stream)),
           "mla_debug_gather_pages")


@dataclass
class DecodeOutputs:
    out: torch.Tensor        # bf16 [N][h][128]
    q_lat: torch.Tensor      # bf16 [N][h][512]
    o_lat: torch.Tensor      # bf16 [N][h][512]
    lse: torch.Tensor        # fp32 [N][h]
    status: torch.Tensor     # int32 [1]


class Decoder:
    """One decode batch shape: plan, workspace and output buffers made once, then
    ``run()`` enqueues absorb -> attention -> combine -> out_uv on the stream.

    Buffers are allocated here by torch (the library allocates nothing).
    """

    def __init__(self, seq_lens, s_q: int, n_heads: int, max_blocks: int, num_blocks: int,
                 device="cuda", scale=None, causal=True, num_clusters: int | None = None,
                 kv_cache: str = "bf16"):
        """``kv_cache``: "bf16" (pool [num_blocks][64][576] bf16) or "fp8" (pool
        uint8 [num_blocks][64][656], see :func:`kv_quantize_fp8`)."""
        if kv_cache not in ("bf16", "fp8"):
            raise ValueError("kv_cache must be 'bf16' or 'fp8'")
        self.kv_cache = kv_cache
        self.seq_lens_host = np.asarray(seq_lens, dtype=np.int32)
        self.B = len(self.seq_lens_host)
        self.s_q, self.H = s_q, n_heads
        self.N = self.B * s_q
        self.dims = make_dims(self.B, s_q, n_heads, max_blocks, num_blocks, scale, causal)
        self.num_clusters = num_clusters or max_clusters()
        self.plan_host, self.num_slots = plan(self.dims, self.seq_lens_host, self.num_clusters)
        dev = torch.device(device)
        self.plan_dev = torch.from_numpy(self.plan_host).to(dev)
        self.seq_lens_dev = torch.from_numpy(self.seq_lens_host).to(dev)
        slots = max(self.num_slots, 1)
        self.o_part = torch.empty(slots * n_heads * 512, dtype=torch.float32, device=dev)   # internal layout
        self.lse_part = torch.empty((slots, n_heads), dtype=torch.float32, device=dev)
        self.q_lat = torch.empty((self.N, n_heads, 512), dtype=torch.bfloat16, device=dev)
        self.o_lat = torch.empty((self.N, n_heads, 512), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((self.N, n_heads), dtype=torch.float32, device=dev)
        self.out = torch.empty((self.N, n_heads, 128), dtype=torch.bfloat16, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.fp8_uk: Fp8Weight | None = None
        self.fp8_uv: Fp8Weight | None = None

    def use_fp8_projections(self, w_uk, w_uv, stream=None):
        """Run the two projections as FP8 block-quantised BMMs from now on:
        W_UK and W_UV are quantised once here (their bf16 copies passed to
        run() are then not read)."""
        self.fp8_uk = quantize_w_uk_fp8(w_uk, stream)
        self.fp8_uv = quantize_w_uv_fp8(w_uv, stream)

    def run(self, q_nope, q_rope, kv_pool, block_table, w_uk, w_uv, stream=None,
            draft_masks=None) -> DecodeOutputs:
        """``draft_masks`` (device int32 [B][s_q], only with causal=False): the
        drafts form a tree, see :func:`decode_attn_tree`."""
        if self.fp8_uk is not None:
            absorb_q_fp8(q_nope, self.fp8_uk, self.q_lat, stream)
        else:
            absorb_q(q_nope, w_uk, self.q_lat, stream)
        if draft_masks is not None and self.kv_cache == "fp8":
            raise ValueError("draft-tree masks need the bf16 cache")
        if self.kv_cache == "fp8":
            decode_attn_fp8cache(self.dims, self.q_lat, q_rope, kv_pool, block_table, self.seq_lens_dev,
                                 self.plan_dev, self.num_clusters, self.o_part, self.lse_part, self.o_lat,
                                 self.lse, self.status, stream)
        elif draft_masks is not None:
            decode_attn_tree(self.dims, self.q_lat, q_rope, kv_pool, block_table, self.seq_lens_dev, draft_masks,
                             self.plan_dev, self.num_clusters, self.o_part, self.lse_part, self.o_lat,
                             self.lse, self.status, stream)
        else:
            decode_attn(self.dims, self.q_lat, q_rope, kv_pool, block_table, self.seq_lens_dev,
                        self.plan_dev, self.num_clusters, self.o_part, self.lse_part, self.o_lat,
                        self.lse, self.status, stream)
        if self.num_slots > 0:
            combine(self.dims, self.plan_dev, self.o_part, self.lse_part, self.o_lat, self.lse, stream)
        if self.fp8_uv is not None:
            out_uv_fp8(self.o_lat, self.fp8_uv, self.out, stream)
        else:
            out_uv(self.o_lat, w_uv, self.out, stream)
        return DecodeOutputs(self.out, self.q_lat, self.o_lat, self.lse, self.status)

    @property
    def launches_per_step(self) -> int:
        return 4 if self.num_slots > 0 else 3


class GraphedStep:
    """One decode step from host memory to host memory, replayed as a CUDA graph.

    For a serving loop with a fixed batch shape: the step's inputs live in
    pinned host buffers (``q_nope``, ``q_rope``, ``block_table``); ``run()``
    replays one graph that copies them to the device, runs absorb ->
    attention -> combine -> out_uv, and copies ``out`` back to the pinned
    ``out`` buffer.  The graph fixes every pointer, so the cache pool, the
    weights and the decoder's buffers must outlive this object; refill the
    host buffers in place between calls.
    """

    def __init__(self, decoder: Decoder, kv_pool, w_uk, w_uv, stream=None):
        dev = kv_pool.device
        N, H = decoder.N, decoder.H
        self.decoder = decoder
        self.q_nope = torch.zeros((N, H, 128), dtype=torch.bfloat16).pin_memory()
        self.q_rope = torch.zeros((N, H, 64), dtype=torch.bfloat16).pin_memory()
        self.block_table = torch.zeros((decoder.B, decoder.dims.max_blocks_per_seq), dtype=torch.int32).pin_memory()
        self.out = torch.empty((N, H, 128), dtype=torch.bfloat16).pin_memory()
        self._q_nope = torch.empty(self.q_nope.shape, dtype=torch.bfloat16, device=dev)
        self._q_rope = torch.empty(self.q_rope.shape, dtype=torch.bfloat16, device=dev)
        self._bt = torch.empty(self.block_table.shape, dtype=torch.int32, device=dev)
        self._args = (kv_pool, w_uk, w_uv)
        self.graph = torch.cuda.CUDAGraph()
        s = stream or torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            self._body()                      # warm-up outside capture (lazy library set-up)
            torch.cuda.synchronize(dev)
            with torch.cuda.graph(self.graph, stream=s):
                self._body()
        torch.cuda.synchronize(dev)

    def _body(self):
        kv_pool, w_uk, w_uv = self._args
        self._q_nope.copy_(self.q_nope, non_blocking=True)
        self._q_rope.copy_(self.q_rope, non_blocking=True)
        self._bt.copy_(self.block_table, non_blocking=True)
        r = self.decoder.run(self._q_nope, self._q_rope, kv_pool, self._bt, w_uk, w_uv)
        self.out.copy_(r.out, non_blocking=True)

    def run(self, sync: bool = True) -> torch.Tensor:
        """Replays the step on the current stream; returns the pinned ``out`` buffer."""
        self.graph.replay()
        if sync:
            torch.cuda.current_stream().synchronize()
        return self.out

    @property
    def h2d_bytes(self) -> int:
        return self.q_nope.nbytes + self.q_rope.nbytes + self.block_table.nbytes

    @property
    def d2h_bytes(self) -> int:
        return self.out.nbytes


class StreamedDecoder:
    """Back-to-back decode steps from pinned host memory to pinned host memory,
    with the copies of one step overlapping the kernels of its neighbours.

    ``depth`` input/output sets rotate: step k uses set i = k % depth.  The user
    fills ``host_in[i]`` (q_nope, q_rope, block_table), calls ``submit()``, and
    reads ``host_out[i]`` once ``ready(i)`` (or ``wait(i)``) says the step's
    device-to-host copy is done.  Three streams carry the work: host-to-device
    copies, the kernels (one CUDA graph per set: absorb -> attention ->
    combine -> out_uv, then a device copy of the output into the set's
    buffer), and device-to-host copies; events keep each set's buffers from
    being overwritten while still in use.  The decoder's scratch buffers are
    shared, so the kernels of consecutive steps run one after another.
    """

    def __init__(self, decoder: Decoder, kv_pool, w_uk, w_uv, depth: int = 2):
        dev = kv_pool.device
        N, H, B = decoder.N, decoder.H, decoder.B
        mb = decoder.dims.max_blocks_per_seq
        self.depth = depth
        self.host_in = [(torch.zeros((N, H, 128), dtype=torch.bfloat16).pin_memory(),
                         torch.zeros((N, H, 64), dtype=torch.bfloat16).pin_memory(),
                         torch.zeros((B, mb), dtype=torch.int32).pin_memory()) for _ in range(depth)]
        self.host_out = [torch.empty((N, H, 128), dtype=torch.bfloat16).pin_memory() for _ in range(depth)]
        self._dev_in = [(torch.empty((N, H, 128), dtype=torch.bfloat16, device=dev),
                         torch.empty((N, H, 64), dtype=torch.bfloat16, device=dev),
                         torch.empty((B, mb), dtype=torch.int32, device=dev)) for _ in range(depth)]
        self._dev_out = [torch.empty((N, H, 128), dtype=torch.bfloat16, device=dev) for _ in range(depth)]
        self._s_in, self._s_cmp, self._s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
        self._ev_in = [torch.cuda.Event() for _ in range(depth)]
        self._ev_cmp = [torch.cuda.Event() for _ in range(depth)]
        self._ev_out = [torch.cuda.Event() for _ in range(depth)]
        self._graphs = []
        self._s_cmp.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(self._s_cmp):
            for i in range(depth):
                qn, qr, bt = self._dev_in[i]
                qn.zero_(); qr.zero_(); bt.zero_()
                decoder.run(qn, qr, kv_pool, bt, w_uk, w_uv)   # warm-up outside capture
                torch.cuda.synchronize(dev)
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=self._s_cmp):
                    r = decoder.run(qn, qr, kv_pool, bt, w_uk, w_uv)
                    self._dev_out[i].copy_(r.out)
                self._graphs.append(g)
        torch.cuda.synchronize(dev)
        self.steps = 0

    def submit(self) -> int:
        """Enqueues the next step on the next set; returns the set index."""
        i = self.steps % self.depth
        reuse = self.steps >= self.depth
        if reuse:   # this set's device inputs are free once its previous step's kernels finished
            self._s_in.wait_event(self._ev_cmp[i])
        with torch.cuda.stream(self._s_in):
            for d, h in zip(self._dev_in[i], self.host_in[i]):
                d.copy_(h, non_blocking=True)
            self._ev_in[i].record(self._s_in)
        self._s_cmp.wait_event(self._ev_in[i])
        if reuse:   # and its device output once its previous copy back finished
            self._s_cmp.wait_event(self._ev_out[i])
        with torch.cuda.stream(self._s_cmp):
            self._graphs[i].replay()
            self._ev_cmp[i].record(self._s_cmp)
        self._s_out.wait_event(self._ev_cmp[i])
        with torch.cuda.stream(self._s_out):
            self.host_out[i].copy_(self._dev_out[i], non_blocking=True)
            self._ev_out[i].record(self._s_out)
        self.steps += 1
        return i

    def input_free(self, i: int) -> bool:
        """``host_in[i]`` may be refilled once its last host-to-device copy is done."""
        return self._ev_in[i].query()

    def ready(self, i: int) -> bool:
        return self._ev_out[i].query()

    def wait(self, i: int) -> torch.Tensor:
        self._ev_out[i].synchronize()
        return self.host_out[i]

    @property
    def streams(self):
        return self._s_in, self._s_cmp, self._s_out


def decode(q_nope, q_rope, kv_pool, block_table, seq_lens, w_uk, w_uv, s_q=1, scale=None,
           causal=True, num_clusters=None) -> DecodeOutputs:
    """One-shot absorbed MLA decode on device tensors (see ``Decoder``)."""
    bt = block_table if isinstance(block_table, torch.Tensor) else torch.as_tensor(block_table)
    bt = bt.to(device=kv_pool.device, dtype=torch.int32).contiguous()
    sl = seq_lens.cpu().numpy() if isinstance(seq_lens, torch.Tensor) else np.asarray(seq_lens)
    d = Decoder(sl, s_q, q_nope.shape[1], bt.shape[1], kv_pool.shape[0], kv_pool.device, scale,
                causal, num_clusters)
    return d.run(q_nope, q_rope, kv_pool, bt, w_uk, w_uv)
