"""bench.py's host logic on CPU: where the roofline denominators come from, when a committed
DRAM-traffic figure may be used, and what the workload description states."""
import json
import os

import pytest

import bench
from top_routing_expert_fp32_b200 import configs


def test_peaks_measured_or_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()            # no file: the recipe's fallback figures
    assert src == "fallback" and peaks == bench.FALLBACK_PEAKS
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6508.8, "bf16_tflops": 1624.0, "bf16_tflops_sustained": 1400.0,
         "other": 1}))
    peaks, src = bench.load_peaks()
    assert src == "measured" and peaks["hbm_gbs"] == 6508.8 and peaks["bf16_tflops"] == 1624.0
    (tmp_path / "MEASURED_PEAKS.json").write_text("{not json")
    assert bench.load_peaks()[1] == "fallback"
    # a file without the sustained figure: the measured ones kept, the missing one named
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6400.0,
                                                              "bf16_tflops": 1600.0}))
    peaks, src = bench.load_peaks()
    assert peaks["hbm_gbs"] == 6400.0 and peaks["bf16_tflops"] == 1600.0
    assert peaks["bf16_tflops_sustained"] == bench.FALLBACK_PEAKS["bf16_tflops_sustained"]
    assert src == "measured (fallback: bf16_tflops_sustained)"
    assert bench.peak_key_source(src, "bf16_tflops_sustained") == "fallback"
    assert bench.peak_key_source(src, "hbm_gbs").startswith("measured")
    assert bench.peak_key_source("fallback", "hbm_gbs") == "fallback"


def test_traffic_used_only_while_the_kernel_sources_are_unchanged(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    entry = {"bytes_per_launch": 123.0, "sources": ["k.cu"],
             "source_sha": bench.source_hash(["k.cu"])}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"up": {"mixtral": entry}}))
    assert bench.traffic_from_profile("up", "mixtral") == 123.0
    assert bench.traffic_from_profile("up", "grok1") is None       # never captured
    assert bench.traffic_from_profile("down", "mixtral") is None
    src.write_text("kernel v2")                                    # the kernel changed since
    assert bench.traffic_from_profile("up", "mixtral") is None


def test_committed_traffic_is_used_exactly_when_its_sources_are_current():
    # Every committed capture names the sources it was taken on; the benchmark reports a
    # capture's bytes only while those sources hash as they did when it was taken, and null
    # otherwise (the kernel has changed since the counters were read).
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        d = json.load(f)
    assert d
    for kernel, per in d.items():
        for workload, e in per.items():
            current = e["source_sha"] == bench.source_hash(e["sources"])
            got = bench.traffic_from_profile(kernel, workload)
            assert got == (e["bytes_per_launch"] if current else None), (kernel, workload)


def test_workload_description_states_the_policies():
    s = bench.workload_desc(configs.CONFIGS["capacity_gshard"])
    assert "N=16384" in s and "E=64" in s and "CF=1.0" in s
    assert "min_capacity=256" in s and "token-major" in s and "renormalised on drops" in s
    s = bench.workload_desc(configs.CONFIGS["decode"], w8=True, packed=True)
    assert "8-bit expert weights" in s and "K-contiguous" in s
    assert "renormalised" in bench.workload_desc(configs.CONFIGS["mixtral"])
    assert "no-renorm" in bench.workload_desc(configs.CONFIGS["grok1"])


def test_reference_arm_runs_exactly_k_sampled_steps(oracle_lib):
    # --impl reference: the oracle on the host, W warm-up and exactly K timed steps, each on a
    # token sample; the line states the sample and whether the rate is extrapolated.
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl",
                        "reference", "--workload", "tiny_f32", "--steps", "3", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, cwd=bench.ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 3 and line["warmup"] == 3
    assert line["value"] > 0 and line["unit"] == "tokens/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    n = line["config"]["sample_tokens_per_step"]
    assert 1 <= n <= 64 and line["extrapolated"] == (n < 64)
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["ms_per_step"] == pytest.approx(1e3 * 64 / line["value"])


def test_table_row_formats_a_line():
    line = {"value": 1.0e6, "ms_per_step": 2.0, "e2e": {"value": 9.0e5},
            "roofline": {"frac": 0.8, "bound": "tensor"},
            "clocks": {"sm_mhz": 1965, "reasons": []},
            "cpu_baseline": {"value": 40.0, "cores": 16},
            "config": {"workload": "mixtral: N=4096", "diagnostics": {
                "balance_loss": 1.0, "drop_rate": 0.0, "load_max_over_mean": 1.02},
                "routing_vs_oracle": {"flips": 0},
                "kernels": {"up": {"TFLOP/s": 1300, "frac_roofline": 0.8},
                            "down": {"TFLOP/s": 1300, "frac_roofline": 0.8},
                            "route": {"ms": 0.01, "frac_hbm": 0.5},
                            "combine": {"ms": 0.02, "frac_hbm": 0.7}}}}
    row = bench.table_row(line)
    assert row.startswith("| mixtral |") and row.count("|") == bench.TABLE_HEAD.split("\n")[0].count("|")
