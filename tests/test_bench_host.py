"""Host-side logic of bench.py on CPU: the FLOP count, the peak lookup, the
traffic figure read from a committed ncu summary, and the clock summary of the
samples taken inside the timed region.
"""

import json
import os

import pytest

import bench
from tiled_online_softmax_03_b200.inputs import WORKLOADS


def test_flops_closed_form():
    w = WORKLOADS["gqa_8k_causal"]
    assert bench.flops(w) == 4.0 * 4 * 32 * 8192 * 8192 * 128 * 0.5
    w = WORKLOADS["bert_large_512_keypad"]
    assert bench.flops(w) == 4.0 * w.B * w.Hq * w.N * w.N * w.d  # non-causal: no halving


def test_peaks_measured_then_fallback(tmp_path, monkeypatch):
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"bf16_tflops": 1700.0,
                                                               "bf16_tflops_sustained": 1400.0}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    burst, sustained, src = bench.peaks()
    assert (burst, sustained) == (1700.0, 1400.0) and src.startswith("measured")
    os.remove(tmp_path / "MEASURED_PEAKS.json")
    burst, sustained, src = bench.peaks()
    assert (burst, sustained) == (bench.FALLBACK_BF16_TFLOPS, bench.FALLBACK_BF16_TFLOPS_SUSTAINED)
    assert src.startswith("fallback")


def write_summary(root, name, sha, dram):
    os.makedirs(root / "profiles", exist_ok=True)
    (root / "profiles" / f"{name}.md").write_text(
        "# summary\n\n## Full capture\n\n"
        f"- kernel_sources_sha256_16: `{sha}`\n- dram_bytes_per_launch: {dram}\n- other: 1\n")


@pytest.mark.parametrize("kind", ["fa_fwd", "fa_fwd_fp8", "fa_bwd"])
def test_recorded_traffic_only_for_the_current_sources(tmp_path, monkeypatch, kind):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_hash", lambda: "0123456789abcdef")
    assert bench.recorded_traffic("gqa_8k_causal", kind) is None  # no summary
    write_summary(tmp_path, f"{kind}_gqa_8k_causal", "0123456789abcdef", 2187983872)
    assert bench.recorded_traffic("gqa_8k_causal", kind) == 2187983872.0
    write_summary(tmp_path, f"{kind}_gqa_8k_causal", "fedcba9876543210", 2187983872)
    assert bench.recorded_traffic("gqa_8k_causal", kind) is None  # taken on other sources


def test_kernel_hash_covers_every_kernel_source():
    names = {os.path.basename(p) for p in bench.KERNEL_SOURCES}
    assert {"fa_fwd_sm100.cu", "fa_ptx.cuh", "fa_schedule.cuh", "fa_bwd_sm100.cuh"} <= names
    assert len(bench.kernel_hash()) == 16


def test_clock_summary_keeps_the_timed_window():
    c = bench.ClockSampler(0)
    line = "0, {sm}, 1965, {pw}, 0x0, {hw}, Not Active, Not Active, {cap}"
    c.rows = [bench.ClockSampler.parse_smi(t, line.format(sm=sm, pw=pw, hw=hw, cap=cap))
              for t, sm, pw, hw, cap in [
                  (1.0, 1965, 300, "Active", "Not Active"),       # before the window
                  (2.0, 1700, 990, "Not Active", "Active"),
                  (2.5, 1650, 1000, "Not Active", "Active"),
                  (3.0, 1680, 995, "Not Active", "Active"),
                  (4.0, 1965, 200, "Not Active", "Not Active")]]  # after
    c.mark(1.5, 3.5)
    s = c.summary()
    assert s["samples"] == 3 and s["sm_mhz"] == 1680 and s["sm_mhz_min"] == 1650
    assert s["reasons"] == ["sw_power_cap"]  # the hw_slowdown sample lies outside the window
    assert s["sm_max_mhz"] == 1965 and s["power_w_median"] == 995
    assert s["window"] == "samples taken inside the timed region"


def test_clock_summary_without_samples():
    c = bench.ClockSampler(0)
    assert bench.ClockSampler.parse_smi(1.0, "garbage") is None
    assert bench.ClockSampler.parse_smi(1.5, "0, n/a, 1965, 1, 0x0, a, b, c, d") is None
    s = c.summary()
    assert s["samples"] == 0 and s["sm_mhz"] is None and s["reasons"] == []


def test_clock_summary_window_without_samples_uses_all():
    c = bench.ClockSampler(0)
    c.rows = [(1.0, 1965.0, 1965.0, 500.0, []), (5.0, 1900.0, 1965.0, 600.0, [])]
    c.mark(2.0, 3.0)  # a region shorter than the sampling period
    s = c.summary()
    assert s["samples"] == 2 and s["window"] == "all samples"
