"""The CUDA arm's JSON line and roofline object, assembled on CPU from fixed stage times.

The stage times are those of the committed full-clip bench line
(profiles/bench_full_clip.md); the line built from them must carry every field
of a bench line and reproduce that run's derived figures.
"""
import json
import types

import pytest

import bench
import oracle.vsa_oracle as O
from vsa_synth import get_config

STAGES = {"pack_pool": 0.68, "score": 0.354, "select": 0.263, "attn": 59.674, "unpack": 0.241}


def _args(**over):
    a = dict(steps=20, warmup=3, sparsity=0.75, fp8=False, config="full", teacher=False)
    a.update(over)
    return types.SimpleNamespace(**a)


def _ks(cfg, s):
    return [O.k_from_sparsity(s, -(-cfg.T // pt) * -(-cfg.H // ph) * -(-cfg.W // pw))
            for (pt, ph, pw) in cfg.tile_shapes]


def _line(args, cfg):
    ks = _ks(cfg, args.sparsity)
    flops = bench.attention_flops(cfg, ks)
    peaks = bench.measured_peaks()
    roof = bench.attn_roofline(args, cfg, peaks, flops, STAGES["attn"])
    ms_step = sum(STAGES.values())
    e2e = {"value": 67.549, "unit": "ms", "h2d_bytes_per_step": 3 * 691273728, "d2h_bytes_per_step": 691273728}
    clocks = {"sm_mhz": 1650.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    stats = {"computed_pairs": 3151, "dense_pairs": 10000}
    return bench.bench_line(args, cfg, 1, ks, flops, ms_step, STAGES, roof, e2e, clocks, stats, []), peaks


def test_line_has_every_key_and_reproduces_the_recorded_run():
    cfg = get_config("full")
    line, peaks = _line(_args(), cfg)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in line, key
    json.dumps(line)
    assert line["metric"] == bench.METRIC and line["unit"] == "ms" and line["higher_is_better"] is False
    assert line["value"] == pytest.approx(sum(STAGES.values()), abs=1e-3)
    assert line["gpu_launches"] == 6 * 20
    r = line["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["algorithmic_flops_per_launch"] == O.attention_flops(cfg, _ks(cfg, 0.75))
    if peaks["source"] == "measured" and peaks["bf16_tflops"] == 1656.9:
        assert r["achieved"] == 821.3 and r["frac"] == 0.4957      # the committed bench line's figures
        assert r["frac_of_sustained_peak"] == 0.5919
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], abs=1e-3)
    traffic = bench.measured_traffic("full", 0.75, 24)
    assert r["traffic"] == traffic
    if traffic is not None:                                        # the capture is of this kernel source
        assert traffic == int((524407040 + 121219072) / 4 * 24)


def test_fp8_line_uses_the_mixed_peak_and_no_traffic():
    cfg = get_config("full")
    line, peaks = _line(_args(fp8=True), cfg)
    r = line["roofline"]
    assert r["peak"] == round(peaks["bf16_tflops"] * 4 / 3, 1)
    assert r["traffic"] is None and "e4m3" in r["peak_kind"]


def test_r2va_line_counts_the_reference_launches():
    cfg = get_config("r2va")
    line, _ = _line(_args(sparsity=cfg.sparsity[0], config="r2va"), cfg)
    assert line["gpu_launches"] == (6 + 4) * 20
    assert "reference segments" in line["config"]["workload"]


def test_clock_summary_reads_nvidia_smi_rows():
    rows = [
        "0, 1980, 1965, 120.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",   # idle
        "0, 1650, 1965, 1005.2, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1665, 1965, 998.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1635, 1965, 1010.9, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "[N/A], garbage",
    ]
    c = bench.summarize_clocks(rows)
    assert c["sm_mhz"] == 1650.0 and c["sm_max_mhz"] == 1965.0 and c["samples"] == 3
    assert c["reasons"] == ["sw_power_cap"] and c["power_w_max"] == 1010.9
    hot = rows[1].replace("Not Active, Not Active, Not Active, Active", "Active, Not Active, Active, Not Active")
    assert bench.summarize_clocks([hot])["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert bench.summarize_clocks([])["reasons"] == ["no samples"]


def test_heads_split_line_is_one_layer_strong_scaling():
    """With the heads of one layer split over 4 ranks, a step is that one layer: the value is the
    slowest rank's step time (not divided by the ranks) and the scaling is strong."""
    cfg = get_config("full")
    args = _args(split="heads")
    ks = _ks(cfg, 0.75)
    flops = bench.attention_flops(cfg, ks)
    roof = bench.attn_roofline(args, cfg, bench.measured_peaks(), flops, STAGES["attn"] / 4)
    line = bench.bench_line(args, cfg, 4, ks, flops, 16.0, STAGES, roof, None, None,
                            {"computed_pairs": 1, "dense_pairs": 2}, [])
    assert line["value"] == 16.0 and line["scaling"] == "strong" and line["n_gpus"] == 4
    assert line["config"]["layers_per_step"] == 1 and "heads" in line["config"]["parallelism"]
    weak = bench.bench_line(_args(), cfg, 4, ks, flops, 16.0, STAGES, roof, None, None,
                            {"computed_pairs": 1, "dense_pairs": 2}, [])
    assert weak["value"] == 4.0 and weak["scaling"] == "weak"


def test_other_workloads_name_their_own_metric():
    assert bench.metric_for(get_config("full")) == bench.METRIC
    m = bench.metric_for(get_config("long"))
    assert "long" in m and "230400" in m
