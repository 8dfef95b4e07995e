"""The allocation-free entry point, checked against the regular one (GPU).

Some callers may not allocate device memory while they run (a serving runtime
that has reserved HBM for its KV-cache pool up front, a plugin called where
cudaMalloc is forbidden).  mla_decode_attn_combine_noalloc serves them: it
takes the host plan and keeps the plan copy and the split-KV partial outputs
in a fixed array inside the library.  Here it must give what
mla_decode_attn + mla_combine give with caller-provided workspace, on two
calls in a row, without any allocation on the torch side.

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

from head_latent_attention_04_b200 import workloads as W
from tests.gpu_helpers import MAX_ABS, REL_FRO, rel_fro

pytestmark = pytest.mark.gpu


def _regular(mla, w, dev):
    """Attention + merge through the entry points that take caller workspace."""
    bt = torch.as_tensor(w.block_table, device=dev)
    wd = w.to(dev)
    d = mla.Decoder(w.seq_lens, w.s_q, w.n_heads, w.max_blocks, w.num_blocks, dev)
    q_lat = mla.absorb_q(wd.q_nope, wd.w_uk)
    mla.decode_attn(d.dims, q_lat, wd.q_rope, wd.kv_pool, bt, d.seq_lens_dev, d.plan_dev, d.num_clusters,
                    d.o_part, d.lse_part, d.o_lat, d.lse, d.status)
    if d.num_slots > 0:
        mla.combine(d.dims, d.plan_dev, d.o_part, d.lse_part, d.o_lat, d.lse)
    torch.cuda.synchronize()
    assert d.status.item() == 0
    return d, q_lat, wd, bt


@pytest.mark.parametrize("case", ["v2_4k", "split_rows", "tiny"])
def test_noalloc_matches_regular_entry_point_twice(case):
    from head_latent_attention_04_b200 import mla
    dev = torch.device("cuda")
    if case == "split_rows":
        w = W.make_workload(5, 2, 128, [3000, 70, 2, 6400, 129], seed=77, pool="scattered:1.5")
    else:
        w = W.preset_workload(case)
    d, q_lat, wd, bt = _regular(mla, w, dev)
    want_o, want_l = d.o_lat.clone(), d.lse.clone()
    assert case == "tiny" or d.num_slots > 0          # the split path is exercised

    o_lat = torch.empty_like(want_o)
    lse = torch.empty_like(want_l)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    before = torch.cuda.memory_allocated(dev)
    for _ in range(2):                                  # the shared array keeps the last call's contents
        o_lat.fill_(float("nan"))
        lse.fill_(float("nan"))
        mla.decode_attn_combine_noalloc(d.dims, q_lat, wd.q_rope, wd.kv_pool, bt, d.seq_lens_dev, d.plan_host,
                                        d.num_clusters, o_lat, lse, status)
        torch.cuda.synchronize()
        assert status.item() == 0
        assert torch.cuda.memory_allocated(dev) == before
        got = o_lat.float().cpu().numpy()
        ref = want_o.float().cpu().numpy()
        assert np.all(np.isfinite(got))
        assert rel_fro(got, ref) <= REL_FRO and float(np.abs(got - ref).max()) <= MAX_ABS
        np.testing.assert_allclose(lse.cpu().numpy(), want_l.cpu().numpy(), rtol=0, atol=2e-2)


def test_noalloc_rejects_batches_beyond_its_array():
    from head_latent_attention_04_b200 import mla
    dev = torch.device("cuda")
    limit = mla.noalloc_scratch_bytes()
    assert limit == 32 << 20
    # two very long rows cut into thousands of pieces: far more partial output than the array holds
    dims = mla.make_dims(2, 1, 128, 1600, 3200)
    plan, slots = mla.plan(dims, [100000, 100000], 2048)
    assert slots * 128 * 512 * 4 > limit
    t = torch.zeros(16, dtype=torch.int32, device=dev)
    with pytest.raises(mla.MlaError) as e:
        mla.decode_attn_combine_noalloc(dims, t, t, t, t, t, plan, 2048, t)
    assert e.value.code == mla.MLA_ERR_WORKSPACE_TOO_SMALL
    assert "scratch" in str(e.value)
