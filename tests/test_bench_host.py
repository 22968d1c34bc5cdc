"""Host-side logic of bench.py (no GPU): the algorithmic byte counts behind the
roofline fractions and the rule that ties an ncu traffic figure to the sources of
its kernel."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads as W  # noqa: E402


def test_fp8_weights_count_one_byte_each():
    cfg = W.CONFIGS["decode"]
    active = 8
    bf16, _, bf16_layer = bench.stage_costs(cfg, active, 1)
    fp8, _, fp8_layer = bench.stage_costs(cfg, active, 1, weight_bytes=1)
    mats = 2  # SwiGLU: gate and up
    assert bf16["expert_up"][1] - fp8["expert_up"][1] == active * mats * cfg.f * cfg.d
    assert bf16["expert_down"][1] - fp8["expert_down"][1] == active * cfg.d * cfg.f
    assert bf16["expert_up"][0] == fp8["expert_up"][0]  # the same flops
    assert bf16_layer - fp8_layer == active * (mats + 1) * cfg.f * cfg.d


def test_stage_bytes_match_the_layer_definition():
    cfg = W.CONFIGS["switch"]  # top-1 ReLU, no shared experts: the down projection writes out itself
    c, flops, layer_bytes = bench.stage_costs(cfg, cfg.m, 1)
    Tk = cfg.T * cfg.k
    assert c["expert_up"][0] == 2.0 * cfg.f * cfg.d * Tk
    assert c["expert_down"][1] == cfg.m * cfg.d * cfg.f * 2 + Tk * cfg.f * 2 + cfg.T * cfg.d * 2
    assert c["combine"][1] == 0.0
    assert layer_bytes == cfg.m * cfg.d * 2 + cfg.m * 2 * cfg.f * cfg.d * 2 + 2 * cfg.T * cfg.d * 2


def test_committed_traffic_is_reported_only_for_unchanged_sources():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as fh:
        t = json.load(fh)
    for workload, stages in t.items():
        for stage, e in stages.items():
            assert e["dram_bytes_per_launch"] > 0 and e["source_files"], (workload, stage)
            current = e["source_hash"] == bench.source_hash(e["source_files"])
            got = bench.traffic_for(workload, stage)
            assert got == (e["dram_bytes_per_launch"] if current else None), (workload, stage)


def test_traffic_goes_null_when_its_kernel_sources_change(tmp_path, monkeypatch):
    csrc = tmp_path / "sparse_mixture_experts_08_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("kernel v1")
    (csrc / "other.cu").write_text("unrelated")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.source_hash(["k.cu"])
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"w": {"s": {"dram_bytes_per_launch": 123.0, "source_hash": h, "source_files": ["k.cu"]}}}))
    assert bench.traffic_for("w", "s") == 123.0
    (csrc / "other.cu").write_text("unrelated, edited")  # another kernel's file: still valid
    assert bench.traffic_for("w", "s") == 123.0
    (csrc / "k.cu").write_text("kernel v2")              # the captured kernel changed: no figure
    assert bench.traffic_for("w", "s") is None
    assert bench.traffic_for("w", "missing") is None


PEAKS = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}


def test_sustained_peak_applies_to_long_or_power_capped_regions():
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    capped = {"sm_mhz": 1330.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    brief_cap = {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    slow_no_reason = {"sm_mhz": 1330.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert not bench.sustained_applies(200, 2.0, full)  # 0.4 s at full clock: the burst peak
    assert bench.sustained_applies(600, 2.0, full)  # over a second of timed steps
    assert bench.sustained_applies(200, 2.4, capped)  # the cap held the clock down
    assert not bench.sustained_applies(200, 2.1, brief_cap)  # capped for a moment, clock near max
    assert not bench.sustained_applies(200, 2.1, slow_no_reason)  # no cap reason: not the cap's regime
    assert not bench.sustained_applies(10, 2.0, None)


def test_contraction_roofline_uses_the_peak_of_its_regime_and_dtype():
    cfg = W.CONFIGS["mixtral"]
    fl, by, ms = 1.924e12, 2.181e9, 1.3  # Mixtral-shaped up projection, 1.3 ms per launch
    burst = bench.roofline_for(cfg, "expert_up", fl, by, ms, PEAKS, "measured", False, False, "none")
    assert burst["bound"] == "tensor" and burst["peak"] == PEAKS["bf16_tflops"]
    assert abs(burst["achieved"] - fl / 1.3e-3 / 1e12) < 1e-9
    assert abs(burst["frac"] - burst["achieved"] / 1600.0) < 1e-12
    assert "frac_of_burst" not in burst
    assert abs(burst["frac_of_nominal_dense"] - burst["achieved"] / 2250.0) < 1e-12
    sus = bench.roofline_for(cfg, "expert_up", fl, by, ms, PEAKS, "measured", True, False, "none")
    assert sus["peak"] == PEAKS["bf16_tflops_sustained"]
    assert abs(sus["frac_of_burst"] - burst["frac"]) < 1e-12  # the same time against the burst figure
    f8 = bench.roofline_for(cfg, "expert_up", fl, by / 2, ms, PEAKS, "measured", False, True, "none")
    assert f8["peak"] == 2 * PEAKS["bf16_tflops"] and f8["nominal_dense_tflops"] == 4500.0
    assert abs(f8["frac"] - burst["frac"] / 2) < 1e-12


def test_weight_streaming_roofline_is_bound_by_hbm():
    cfg = W.CONFIGS["decode"]  # 16 tokens: a few flops per weight byte, far below the ridge point
    fl, by, ms = 7.5e9, 1.88e9, 0.31
    r = bench.roofline_for(cfg, "expert_up", fl, by, ms, PEAKS, "measured", False, False, "none")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == PEAKS["hbm_gbs"]
    assert abs(r["achieved"] - by / 0.31e-3 / 1e9) < 1e-6
    assert r["traffic"] is None  # no committed capture under this key


def test_reference_arm_prints_the_config_of_the_gpu_arm(capsys):
    """Both arms describe the same run in `config`, so a comparison of the two lines
    compares like with like; the oracle's own execution goes under `execution`."""
    import argparse

    args = argparse.Namespace(config="tiny", steps=1, warmup=3, gpus=1)
    assert bench.reference_arm(args) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 1 and line["warmup"] == 3
    assert line["config"] == bench.run_config(W.CONFIGS["tiny"], 1)
    assert line["e2e"]["value"] == line["value"] == line["cpu_baseline"]["value"]
    assert line["execution"]["l2"] == "n/a (CPU)"


def test_profiles_index_lists_every_summary_and_each_gives_its_command():
    pdir = os.path.join(ROOT, "profiles")
    with open(os.path.join(pdir, "README.md")) as fh:
        index = fh.read()
    summaries = sorted(f for f in os.listdir(pdir) if f.endswith(".md") and f != "README.md")
    for f in summaries:
        assert f"`{f}`" in index, f"{f} is not in profiles/README.md"
        with open(os.path.join(pdir, f)) as fh:
            text = fh.read()
        assert "ncu " in text and "--clock-control none" in text, f"{f} gives no ncu command"
        assert "python bench.py" in text, f"{f} does not name the committed command it profiled"
    for f in os.listdir(pdir):  # summaries only: no raw reports or scripts
        assert f.endswith((".md", ".txt", ".json")), f
