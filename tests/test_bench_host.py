"""Host-side logic of bench.py: the algorithmic byte counts behind the roofline
fractions, the traffic record lookup and the clock-sample summary.  No GPU."""
import json
import os
import tempfile

import pytest

import bench


def test_algorithmic_bytes_of_the_workloads():
    # prefill: six bf16 inputs and bf16 y per head-token (14 * 64 B = 896 B),
    # fp32 s0 in and sT out per head (32 KiB): 947.9 MB
    assert bench.fwd_bytes(8, 4096, 32) == 8 * 4096 * 32 * 896 + 8 * 32 * 32768 == 947_912_704
    # backward: six inputs and dy read, six bf16 gradients written (1664 B per
    # head-token), s0 in and ds0 out: 1.753 GB
    assert bench.bwd_bytes(8, 4096, 32) == 8 * 4096 * 32 * 1664 + 8 * 32 * 32768 == 1_753_219_072
    # decode step: the fp32 state read and written (32 KiB per head) plus six
    # inputs and y (896 B per head): 344.7 MB per step
    assert bench.step_bytes(256, 40) == 256 * 40 * (32768 + 896) == 344_719_360


def test_fp32_peak_is_derived_from_the_clock():
    # 148 SMs x 128 FP32 lanes x 2 flop per FMA at 1965 MHz
    assert bench.fp32_peak_tflops(1965.0) == pytest.approx(74.44992)


def test_recorded_traffic_only_for_the_source_it_was_taken_on():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    srcs = {"fwd_chunk": ("fwd_chunk.cu", "umma.cuh", "common.cuh"),
            "fwd_chunk_timemix": ("fwd_chunk.cu", "umma.cuh", "common.cuh"),
            "fwd_seq": ("fwd_seq.cu", "umma.cuh", "common.cuh"),
            "step": ("step.cu", "common.cuh")}
    for kernel, names in srcs.items():
        entry = rec[kernel]
        assert entry["dram_bytes_per_launch"] > 0 and entry["profile"].startswith("profiles/")
        assert os.path.exists(os.path.join(bench.ROOT, entry["profile"]))
        got = bench.recorded_traffic(kernel, entry["source_hash"])
        assert got == entry["dram_bytes_per_launch"]
        assert bench.recorded_traffic(kernel, "0" * 16) is None
        # the hash is over the named sources, in order
        assert len(bench.source_hash(*names)) == 16
    assert bench.recorded_traffic("no_such_kernel", "0" * 16) is None


def _summary_of(lines):
    s = bench.ClockSampler("GPU-test")
    fd, s.path = tempfile.mkstemp(suffix=".csv")
    with os.fdopen(fd, "w") as f:
        f.write("\n".join(lines) + "\n")
    return s.summary()


def test_clock_summary_median_of_busy_samples_and_reasons():
    rows = ["1965, 1965, 350.5, 0x0, Not Active, Not Active, Not Active, Not Active",
            "1965, 1965, 371.7, 0x0, Not Active, Not Active, Not Active, Not Active",
            "1950, 1965, 402.0, 0x4, Not Active, Not Active, Not Active, Active",
            "345, 1965, 90.0, 0x0, Not Active, Not Active, Not Active, Not Active",   # idle sample
            "garbage line"]
    out = _summary_of(rows)
    assert out["samples"] == 4
    assert out["sm_mhz"] == 1965.0          # the idle 345 MHz sample is not counted as load
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]
    assert out["power_w_max"] == pytest.approx(402.0)


def test_clock_summary_flags_slowdowns_and_missing_samples():
    rows = ["1400, 1965, 600.0, 0x8, Active, Not Active, Active, Not Active"]
    out = _summary_of(rows)
    assert out["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert out["sm_mhz"] == 1400.0
    assert _summary_of([])["reasons"] == ["unsampled"]
