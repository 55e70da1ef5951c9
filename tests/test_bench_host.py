"""Host-side logic of bench.py (no GPU): byte and launch accounting, clock-sample parsing, the rule that a
committed DRAM-traffic figure is used only for the kernel sources it was measured on, and the shape of the
reference arm's JSON line."""
import json
import os
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from ar_lm_decoding_b200 import synth  # noqa: E402


def test_algorithmic_bytes_closed_form():
    cfg = synth.CONFIGS["qwen3-8b_k8"]
    psum = cfg.B * cfg.P
    b = bench.algorithmic_bytes(cfg, psum)
    # one layer: every cached key and value row once (2 x Hkv x D bf16 each), the step's Q / K_new / V_new read
    # and O (bf16) / LSE (f32) written once
    per_layer = 2 * 2 * cfg.Hkv * cfg.D * cfg.P + cfg.R * (2 * cfg.Hq * cfg.D + 2 * 2 * cfg.Hkv * cfg.D
                                                            + 2 * cfg.Hq * cfg.D + 4 * cfg.Hq)
    assert (b["kv"] + b["qkvo"]) // cfg.L == per_layer == 18425856
    # verify and draft selection: the p and q rows of the k slots and the k slot rows of group j*, bf16
    assert b["logits"] == 3 * cfg.k * cfg.V * 2
    assert bench.attn_flops(cfg, psum) == 4 * cfg.L * cfg.Hq * cfg.R * cfg.D * cfg.P


def test_kernels_per_step():
    cfg = synth.CONFIGS["qwen3-8b_k8"]
    assert bench.kernels_per_step(cfg) == cfg.L + 1  # L attention launches, verify + commit (1)


def test_clock_sample_parsing():
    rows = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1950, 1965, 820.4, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1890, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "garbage line",
        "0, N/A, 1965, 0, 0, Not Active, Not Active, Not Active, Not Active",
    ]
    c = bench.parse_clock_samples("\n".join(rows))
    assert c["samples"] == 3 and c["sm_mhz"] == 1950 and c["sm_max_mhz"] == 1965
    assert c["reasons"] == ["sw_power_cap"]
    assert bench.parse_clock_samples("")["reasons"] == ["no samples"]


def test_traffic_figure_only_for_matching_sources(tmp_path, monkeypatch):
    csrc = tmp_path / "ar_lm_decoding_b200" / "csrc"
    csrc.mkdir(parents=True)
    for n in ("attn_sm100.cu", "attn.cuh", "common.cuh", "tc.cuh", "verify.cu"):
        (csrc / n).write_text(f"// {n}\nint x_{n.replace('.', '_')} = 1;\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    cfg = synth.CONFIGS["qwen3-8b_k8"]
    rec = {"workload": cfg.name, "dram_bytes_per_launch": 123, "source_sha256": bench.kernel_source_hash()}
    path = tmp_path / "profiles" / "attn_traffic.json"
    path.write_text(json.dumps(rec))
    assert bench.load_traffic(cfg) == 123
    assert bench.load_traffic(synth.CONFIGS["qwen2.5-1.5b_k4"]) is None  # another workload
    (csrc / "verify.cu").write_text("int changed = 2;\n")  # not an attention source: the figure stands
    assert bench.load_traffic(cfg) == 123
    (csrc / "tc.cuh").write_text("/* a new comment */ // and another\nint   x_tc_cuh =\n 1;\n")  # comments, layout
    assert bench.load_traffic(cfg) == 123
    (csrc / "tc.cuh").write_text("int x_tc_cuh = 2;\n")  # the attention kernel's code changed: no figure
    assert bench.load_traffic(cfg) is None
    path.write_text("{not json")
    assert bench.load_traffic(cfg) is None


def test_reference_arm_line():
    import oracle
    oracle.build()
    cfg = synth.CONFIGS["tiny"]
    args = types.SimpleNamespace(steps=2, warmup=1)
    res = bench.reference_arm(args, cfg)
    assert res["impl"] == "reference" and res["metric"] == bench.METRIC and res["unit"] == bench.UNIT
    assert res["value"] > 0 and res["higher_is_better"] is True
    assert res["cpu_baseline"]["kind"] == "oracle" and res["cpu_baseline"]["value"] == res["value"]
    assert res["e2e"] == {"value": res["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}
    json.dumps(res)


def test_line_sanity_rules():
    line = {"value": 1000.0, "ms_per_step": 1.0, "steps": 10, "gpu_launches": 380,
            "roofline": {"us_per_launch": 20.0}, "e2e": {"value": 500.0}}
    bench.check_line(line)
    with pytest.raises(AssertionError):  # end to end cannot beat the device-only rate
        bench.check_line({**line, "e2e": {"value": 1500.0}})
    with pytest.raises(AssertionError):  # 36 attention launches of 30 us do not fit a 1 ms step
        bench.check_line({**line, "roofline": {"us_per_launch": 30.0}})


def test_cpu_baseline_reports_single_thread_and_all_cores():
    import oracle
    oracle.build()
    cb = bench.cpu_baseline(synth.CONFIGS["tiny"], 0.2)
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["cores"] >= 1
    assert cb["single_thread"]["threads"] == 1 and cb["single_thread"]["value"] > 0
    assert cb["host"]["nproc"] >= 1 and cb["host"]["cpu_model"]


def test_copy_groups_cover_every_layer_once():
    """The end-to-end leg's host-to-device copy groups: consecutive, covering layers 0..L-1 exactly once, sized
    1, 2, 4, 8, 8, ... (the last takes the rest), never more than the cap."""
    for L in (1, 2, 3, 7, 28, 36, 64, 80):
        for cap in (1, 4, 8, 16):
            groups = bench.copy_groups(L, cap=cap)
            assert groups[0][0] == 0 and groups[-1][1] == L
            assert all(a[1] == b[0] for a, b in zip(groups, groups[1:]))
            sizes = [b - a for a, b in groups]
            assert all(0 < s <= cap for s in sizes)
            for i, s in enumerate(sizes[:-1]):
                assert s == min(cap, 2 ** i)
