"""CPU pieces of bench.py: the fairer float32 absorbed-order CPU figure computes
the same attention as the oracle, and the algorithmic accounting matches the
formulas the measurement uses."""
import json

import numpy as np

import bench
from head_latent_attention_04_b200 import workloads as W
from oracle import mla_oracle as O


def test_cpu_absorbed_fp32_matches_oracle():
    w = W.make_workload(3, 2, 8, [5, 70, 130], seed=4)
    for b in range(w.B):
        rows = slice(b * w.s_q, (b + 1) * w.s_q)
        ref = O.mla_decode(w.q_nope[rows].double().numpy(), w.q_rope[rows].double().numpy(),
                           [w.cache_rows(b).double().numpy()], w.w_uk.double().numpy(),
                           w.w_uv.double().numpy(), w.s_q, with_intermediates=False)["out"]
        got = bench.cpu_absorbed_fp32(w, b)
        np.testing.assert_allclose(got, ref, rtol=2e-4, atol=2e-5)


def test_algorithmic_accounting():
    acc = bench.algorithmic([4096] * 32, 1, 128)
    assert acc["cache_bytes"] == 32 * 4096 * 1152
    assert acc["attn_flops"] == 32 * 4096 * 2 * 128 * (2 * 512 + 64)
    assert acc["attn_bytes"] == 32 * 4096 * 1152 + 32 * 128 * (576 + 512) * 2
    # causal MTP: query i of a sequence of length T attends T - 1 + i keys
    acc2 = bench.algorithmic([10, 20], 2, 128)
    assert acc2["attn_flops"] == (9 + 10 + 19 + 20) * 2 * 128 * (2 * 512 + 64)


def test_algorithmic_accounting_fp8_weights():
    """E4M3 weights: one byte per element plus one fp32 scale per 128 x 128 block."""
    bf = bench.algorithmic([4096] * 32, 1, 128)
    f8 = bench.algorithmic([4096] * 32, 1, 128, weight_bytes=1)
    assert bf["step_bytes"] - f8["step_bytes"] == 2 * 512 * 128 * 128 - 2 * 4 * 128 * 4
    assert f8["attn_bytes"] == bf["attn_bytes"] and f8["step_flops"] == bf["step_flops"]


def test_algorithmic_accounting_fp8_cache():
    """FP8 latent cache: 656 bytes per cached token (512 codes, 4 fp32 scales,
    64 bf16 k_rope) instead of 1152; the products are unchanged."""
    bf = bench.algorithmic([4096] * 32, 1, 128)
    f8 = bench.algorithmic([4096] * 32, 1, 128, cache_row_bytes=656)
    assert 656 == 512 + 4 * 4 + 64 * 2
    assert f8["cache_bytes"] == 32 * 4096 * 656
    assert bf["attn_bytes"] - f8["attn_bytes"] == 32 * 4096 * (1152 - 656)
    assert f8["attn_flops"] == bf["attn_flops"]


def test_next_path_roofline_picks_the_binding_unit():
    peaks = {"hbm_gbs": 6545.0, "bf16_tflops": 1630.1, "bf16_tflops_sustained": 1374.1}
    # 30.3 MB and 7.75 GFLOP: 4.6 us of HBM against 4.8 us of tensor time -> tensor
    r = bench._roof(7.75e9, 30.3e6, 0.010, peaks, "measured")
    assert r["bound"] == "tensor" and abs(r["achieved"] - 775.0) < 1e-6 and abs(r["frac"] - 775.0 / 1630.1) < 1e-9
    r = bench._roof(1e6, 30.3e6, 0.010, peaks, "measured")
    assert r["bound"] == "hbm" and abs(r["achieved"] - 3030.0) < 1e-6


def test_draft_tree_inputs_are_ancestor_masks():
    # the spec path's seeded trees: every mask is the oracle's visibility set of its parents
    parents, masks = W.draft_tree(6, 8, 4)
    assert masks.dtype == np.int32 and masks.shape == (6, 8)
    for b in range(6):
        assert parents[b][0] == -1 and all(-1 <= p < i for i, p in enumerate(parents[b]))
        assert [int(m) for m in masks[b]] == O.tree_masks(parents[b])
    # a different seed draws other trees; the same seed the same ones
    assert W.draft_tree(6, 8, 4)[0] == parents and W.draft_tree(6, 8, 5)[0] != parents


def test_spec_path_arguments():
    a = bench.parse_args(["--path", "spec", "--s-q", "4", "--draft", "chain"])
    assert (a.path, a.s_q, a.draft) == ("spec", 4, "chain")
    a = bench.parse_args(["--path", "spec"])
    assert (a.s_q, a.draft) == (8, "tree")


def test_visible_keys_count_the_oracle_visibility():
    # the spec path's FLOP count: per query row, the keys the oracle's mask keeps
    parents, masks = W.draft_tree(3, 5, 11)
    lens = [5, 9, 70]
    got = bench.visible_keys(lens, 5, masks)
    want = []
    for b, T in enumerate(lens):
        for i in range(5):
            keep = [t < T - 5 or (masks[b][i] >> (t - (T - 5))) & 1 for t in range(T)]
            want.append(int(sum(bool(k) for k in keep)))
    assert got == want
    # a chain is the causal rule, and the causal count is what algorithmic() charges
    chain = np.array([O.tree_masks([-1, 0, 1, 2, 3])] * 3, dtype=np.int32)
    assert bench.visible_keys(lens, 5, chain) == bench.visible_keys(lens, 5)
    assert sum(bench.visible_keys(lens, 5)) == bench.algorithmic(lens, 5, 16)["pairs"]


def test_reference_arm_line(monkeypatch, capsys):
    # the reference arm times the oracle on the host: one JSON line on rank 0
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    bench.main(["--impl", "reference", "--config", "tiny", "--steps", "2", "--warmup", "1"])
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"]
    assert d["config"]["workload"] == "tiny" and d["steps"] == 2 and d["n_gpus"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_print_nothing(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--config", "tiny", "--steps", "2", "--warmup", "1"])
    assert capsys.readouterr().out.strip() == ""


def test_clock_summary_segments():
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.ok, cs.samples, cs.reasons, cs.max_mhz = True, [1965, 1965, 1900, 1800, 1700], 0x4, 1965
    out = cs.summary({"steps": (0, 2), "attention": (2, None)})
    assert out["sm_mhz"] == 1900 and out["reasons"] == ["sw_power_cap"]
    assert out["segments"] == {"steps": {"sm_mhz": 1965.0, "samples": 2}, "attention": {"sm_mhz": 1800.0, "samples": 3}}
