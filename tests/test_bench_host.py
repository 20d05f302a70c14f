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


def test_committed_traffic_matches_the_current_sources():
    # Every committed capture names the sources it was taken on; the ones the benchmark reads
    # for its default line must hash to the current files.
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        d = json.load(f)
    e = d["up"]["mixtral"]
    assert e["source_sha"] == bench.source_hash(e["sources"])
    assert bench.traffic_from_profile("up", "mixtral") == e["bytes_per_launch"]


def test_workload_description_states_the_policies():
    s = bench.workload_desc(configs.CONFIGS["capacity_gshard"])
    assert "N=16384" in s and "E=64" in s and "CF=1.0" in s
    assert "min_capacity=256" in s and "token-major" in s and "renormalised on drops" in s
    s = bench.workload_desc(configs.CONFIGS["decode"], w8=True, packed=True)
    assert "8-bit expert weights" in s and "K-contiguous" in s
    assert "renormalised" in bench.workload_desc(configs.CONFIGS["mixtral"])
    assert "no-renorm" in bench.workload_desc(configs.CONFIGS["grok1"])
