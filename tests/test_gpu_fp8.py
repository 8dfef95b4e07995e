"""FP8 block-quantised projections on the GPU against the FP8 oracle.

The quantisers are compared code by code and scale by scale (a float32
decision on both sides); the BMMs within the tolerance of the bf16 path
(relative Frobenius <= 5e-3 and max abs <= 2e-2), against the oracle's
float64 product of the oracle's own codes."""
import numpy as np
import pytest
import torch

from head_latent_attention_04_b200 import workloads as W
from oracle import fp8 as F
from tests.gpu_helpers import check_out, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mla():
    from head_latent_attention_04_b200 import mla as m
    return m


def _codes(t: torch.Tensor) -> np.ndarray:
    return F.e4m3_decode(t.cpu().numpy())


@pytest.mark.parametrize("H", [1, 7, 128])
def test_weight_quantisation_is_bit_exact(mla, H):
    w = W.make_workload(1, 1, H, [1], seed=H)
    wuk, wuv = w.w_uk.cuda(), w.w_uv.cuda()
    wuv[:128, 0, :] = 0                                    # an all-zero block takes scale 1
    qk, qv = mla.quantize_w_uk_fp8(wuk), mla.quantize_w_uv_fp8(wuv)
    torch.cuda.synchronize()
    ok_codes, ok_s = F.quantize_w_uk(wuk.float().cpu().numpy())
    ov_codes, ov_s = F.quantize_w_uv(wuv.float().cpu().numpy())
    assert np.array_equal(_codes(qk.codes), ok_codes)
    assert np.array_equal(qk.scales.cpu().numpy(), ok_s)
    assert np.array_equal(_codes(qv.codes), ov_codes)
    assert np.array_equal(qv.scales.cpu().numpy(), ov_s)
    assert qv.scales[0, 0].item() == 1.0 and int(qv.codes[0, :, :128].int().sum()) == 0


def test_row_quantisation_is_bit_exact(mla):
    g = torch.Generator().manual_seed(7)
    x = torch.randn((37, 3, 512), generator=g)
    x[0, 0, :128] = 0                                      # zero vector
    x[1, 1, 128:256] *= 1e-4                               # codes in the subnormal range
    x[2, 2, 256:384] *= 1e4
    x[3, 0, 384:] = torch.linspace(-5, 5, 128)             # many exact ties after scaling
    xb = x.to(torch.bfloat16)
    codes, scales = mla.quantize_rows_fp8(xb.cuda())
    torch.cuda.synchronize()
    want_c, want_s = F.quantize_act(xb.float().numpy())
    assert np.array_equal(_codes(codes), want_c)
    assert np.array_equal(scales.cpu().numpy(), want_s)


def _weights(H, seed):
    w = W.make_workload(1, 1, H, [1], seed=seed)
    return w.w_uk, w.w_uv


@pytest.mark.parametrize("N,H", [(1, 1), (2, 16), (37, 128), (64, 128), (100, 9), (256, 128), (300, 7)])
def test_absorb_q_fp8_matches_oracle(mla, N, H):
    wuk, _ = _weights(H, N + H)
    g = torch.Generator().manual_seed(N)
    q = torch.randn((N, H, 128), generator=g).to(torch.bfloat16)
    wq = mla.quantize_w_uk_fp8(wuk.cuda())
    got = mla.absorb_q_fp8(q.cuda(), wq)
    torch.cuda.synchronize()
    codes, s = F.quantize_w_uk(wuk.float().numpy())
    want = F.absorb_fp8(q.float().numpy(), codes, s)
    check_out(got, want)


@pytest.mark.parametrize("N,H", [(1, 1), (2, 16), (37, 128), (128, 128), (130, 3), (300, 7)])
def test_out_uv_fp8_matches_oracle(mla, N, H):
    _, wuv = _weights(H, N + 2 * H)
    g = torch.Generator().manual_seed(N + 7)
    o = (torch.randn((N, H, 512), generator=g) * 0.05).to(torch.bfloat16)
    o[0, 0, 128:256] = 0                                   # a zero vector (scale 1, zero codes)
    wq = mla.quantize_w_uv_fp8(wuv.cuda())
    got = mla.out_uv_fp8(o.cuda(), wq)
    torch.cuda.synchronize()
    codes, s = F.quantize_w_uv(wuv.float().numpy())
    want = F.out_uv_fp8(o.float().numpy(), codes, s)
    check_out(got, want)


@pytest.mark.parametrize("N,H", [(37, 128), (300, 5)])
def test_fp8_projections_write_only_their_rows(mla, N, H):
    wuk, wuv = _weights(H, N)
    g = torch.Generator().manual_seed(N + 1)
    q = torch.randn((N, H, 128), generator=g).to(torch.bfloat16).cuda()
    o = (torch.randn((N, H, 512), generator=g) * 0.05).to(torch.bfloat16).cuda()
    big_q = torch.full((N + 40, H, 512), 3.0, dtype=torch.bfloat16, device="cuda")
    big_o = torch.full((N + 40, H, 128), 3.0, dtype=torch.bfloat16, device="cuda")
    mla.absorb_q_fp8(q, mla.quantize_w_uk_fp8(wuk.cuda()), big_q[:N])
    mla.out_uv_fp8(o, mla.quantize_w_uv_fp8(wuv.cuda()), big_o[:N])
    torch.cuda.synchronize()
    assert bool((big_q[N:] == 3.0).all()) and bool((big_o[N:] == 3.0).all())
    ck, sk = F.quantize_w_uk(wuk.float().numpy())
    cv, sv = F.quantize_w_uv(wuv.float().numpy())
    check_out(big_q[:N], F.absorb_fp8(q.float().cpu().numpy(), ck, sk))
    check_out(big_o[:N], F.out_uv_fp8(o.float().cpu().numpy(), cv, sv))


def test_fp8_step_against_bf16_step(mla):
    """The v2_4k step with FP8 projections: its output differs from the bf16
    step's by the quantisation error only (a few percent), and its q_lat
    matches the FP8 oracle."""
    w = W.preset_workload("v2_4k", device="cuda")
    bt = torch.as_tensor(w.block_table, device="cuda")
    dec = mla.Decoder(w.seq_lens, w.s_q, w.n_heads, w.max_blocks, w.num_blocks, torch.device("cuda"))
    ref = dec.run(w.q_nope, w.q_rope, w.kv_pool, bt, w.w_uk, w.w_uv).out.float().clone()
    dec.use_fp8_projections(w.w_uk, w.w_uv)
    got = dec.run(w.q_nope, w.q_rope, w.kv_pool, bt, w.w_uk, w.w_uv)
    torch.cuda.synchronize()
    assert int(dec.status.item()) == 0
    err = rel_fro(got.out.float().cpu().numpy(), ref.cpu().numpy())
    assert 1e-3 < err < 0.08, err
    codes, s = F.quantize_w_uk(w.w_uk.float().cpu().numpy())
    want_q = F.absorb_fp8(w.q_nope.float().cpu().numpy(), codes, s)
    check_out(got.q_lat, want_q)
