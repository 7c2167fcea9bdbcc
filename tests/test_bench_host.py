"""Host-side pieces of bench.py (CPU): algorithmic byte counts, the ncu traffic record and its source-hash gate,
the measured peaks, and the decoding of NVML clock-event reasons."""
import json
import os

import bench
from exact_io_aware_48_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_recorded_traffic_matches_the_current_sources():
    # the committed record was taken on the recorded kernels' sources as they are now (editing them means retaking it)
    with open(os.path.join(ROOT, "profiles", "kernel_traffic.json")) as f:
        rec = json.load(f)
    assert rec["src_hash"] == bench.kernel_src_hash()


def test_algorithmic_bwd_bytes_closed_form():
    # GPT-2 shape B8 H12 N1024 d64: Q, K, V, dO read and dK, dV written (6 tensors of B*H*N*d 16-bit values) plus
    # the fp32 LSE2 and D rows of the 128-padded row space
    w = inputs.workloads()["gpt2"]
    assert bench.algorithmic_bwd_bytes(w) == 6 * 8 * 12 * 1024 * 64 * 2 + 2 * 4 * 8 * 12 * 8 * 128 == 76283904


def test_recorded_traffic_is_gated_by_the_source_hash(monkeypatch):
    with open(os.path.join(ROOT, "profiles", "kernel_traffic.json")) as f:
        rec = json.load(f)
    e = rec["lc16k"]["bwd_kernel<128,bf16>"]
    monkeypatch.setattr(bench, "kernel_src_hash", lambda: rec["src_hash"])
    assert bench.recorded_traffic("lc16k", "bwd_kernel<128,bf16>") == e["read"] + e["write"]
    assert bench.recorded_traffic("lc16k", "no_such_kernel") is None
    monkeypatch.setattr(bench, "kernel_src_hash", lambda: "0" * 16)
    assert bench.recorded_traffic("lc16k", "bwd_kernel<128,bf16>") is None


def test_peaks_come_from_the_measured_file():
    # the driver writes MEASURED_PEAKS.json on the machines it measured; without it the recipe's fallback is used
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    burst, sustained, hbm, src = bench.peaks()
    if not os.path.exists(path):
        assert (burst, sustained, hbm, src) == (1590.0, 1400.0, 6650.0, "fallback")
        return
    with open(path) as f:
        p = json.load(f)
    assert (burst, sustained, hbm, src) == (float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]),
                                            float(p["hbm_gbs"]), "measured")


def test_clock_reasons_are_decoded_and_idle_is_ignored():
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.ok, cs.max_mhz = True, 1965
    cs.samples = [1965, 1800, 1700]
    cs.reasons = 0x1 | 0x4 | 0x40  # gpu_idle, sw_power_cap, hw_thermal_slowdown
    s = cs.summary()
    assert s["sm_mhz"] == 1800 and s["sm_max_mhz"] == 1965 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap", "hw_thermal_slowdown"]
    cs.ok = False
    assert cs.summary()["reasons"] == ["nvml unavailable"]
