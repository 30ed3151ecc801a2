"""Host-side pieces of bench.py (CPU only): the roofline byte counts, the clock
sampler's windowing and the peak / traffic lookups."""
import json

import pytest
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def test_full_stream_bytes_config3():
    # K draft rows + K+1 target rows of bf16 logits, W once, the gathered U rows
    w = synth.WORKLOADS["c3"]
    assert bench.full_stream_bytes(w) == 2 * 64 * 33 * 129280 + 2 * 256 * 129280 + 2 * 64 * 16 * 256
    assert bench.full_stream_bytes(w) == 612794368


def test_early_exit_bytes_bounds():
    w = synth.WORKLOADS["c3"]
    full = bench.full_stream_bytes(w)
    assert bench.early_exit_bytes(w, np.full(w.B, w.K + 1)) == full
    one = bench.early_exit_bytes(w, np.ones(w.B, dtype=np.int64))
    assert one == 2 * (w.B * w.K + w.B) * w.V + 2 * w.r * w.V + 2 * w.B * w.K * w.r
    assert one < full


def test_clock_sampler_keeps_the_timed_window_only():
    c = bench.ClockSampler(0)
    row = lambda mhz, reason: ["0", str(mhz), "1965", "300.0", "0x0", "Not Active", "Not Active",
                               "Not Active", reason]
    c.samples = [(1.0, row(900, "Not Active")), (2.0, row(1965, "Not Active")),
                 (3.0, row(1950, "Active")), (9.0, row(600, "Not Active"))]
    c.t0, c.t1 = 1.5, 3.5
    s = c.summary()
    assert s["samples"] == 2
    assert s["sm_mhz"] == (1965 + 1950) / 2
    assert s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_sampler_without_samples_says_so():
    c = bench.ClockSampler(0)
    c.t0, c.t1 = 0.0, 1.0
    assert c.summary()["reasons"] == ["unsampled"]


def test_measured_peak_reads_the_driver_file():
    peak, kind = bench.measured_peak()
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        assert kind == "measured" and peak == float(json.load(open(p))["hbm_gbs"])
    else:
        assert kind == "fallback" and peak == 6650.0


@pytest.mark.parametrize("name", ["k_cycle_tc_c3", "k_verify_ee_c3"])
def test_recorded_traffic_only_for_the_profiled_source(name):
    assert bench.recorded_traffic("not-the-profiled-source", name) is None
    p = os.path.join(ROOT, "profiles", f"{name}_ncu.json")
    d = json.load(open(p))
    assert bench.recorded_traffic(d["csrc_hash"], name) == d["dram_bytes_per_launch"]


def test_clock_sampler_short_region_takes_the_nearest_samples():
    # a timed region shorter than the sampling period: the samples on each side
    c = bench.ClockSampler(0)
    row = lambda mhz: ["0", str(mhz), "1965", "300.0", "0x0", "Not Active", "Not Active",
                       "Not Active", "Not Active"]
    c.samples = [(1.0, row(1900)), (2.0, row(1965)), (3.0, row(1950)), (4.0, row(1000))]
    c.t0, c.t1 = 2.2, 2.3
    s = c.summary()
    assert s["samples"] == 2 and s["sm_mhz"] == (1965 + 1950) / 2
    assert "nearest" in s["window"]


def test_w_l2_bytes_counts_the_streamed_chunks():
    # V = 129280: 1010 chunks of 128 tokens, 7 per CTA on 148 SMs (145 CTAs, the
    # last with 2); 3 chunks per CTA stay in tensor memory, the rest stream every
    # MMA round (16 draft steps + the final step)
    w = synth.WORKLOADS["c3"]
    streamed = 144 * (7 - 3) + 0
    assert bench.w_l2_bytes(w, 148) == streamed * 128 * 256 * 2 * 17
    assert bench.w_l2_bytes(w, 148, greedy=True) == streamed * 128 * 256 * 2 * 16


def test_near_threshold_counts_flagged_and_mismatched_rows():
    K = 3
    # row 0: a draft flag after its stop row (position 2 > stop 1) does not count;
    # row 1: all accepted, last token differs (mismatch); row 2: flagged at the stop row
    ref = {"tau": np.array([2, 4, 1]), "out": np.array([[5, 6, -1, -1], [1, 2, 3, 4], [9, -1, -1, -1]]),
           "flag_draft": np.array([2, 3, 0]), "flag_accept": np.array([3, 3, 3]),
           "flag_final": np.array([0, 0, 0])}
    out = np.array([[5, 6, -1, -1], [1, 2, 3, 7], [8, -1, -1, -1]])
    tau = np.array([2, 4, 1])
    r = bench.near_threshold(ref, out, tau, K)
    assert r == {"rows_checked": 3, "flagged": 1, "mismatched_unflagged": 1}


def test_kernel_hash_follows_code_not_comments(tmp_path):
    """A recorded traffic figure is keyed on the profiled kernel's own source
    and the shared headers: comments and other kernels' files do not change
    the key, a code change in the kernel's file does."""
    import shutil
    src = os.path.join(ROOT, "draft_sampling_verification_head_b200", "csrc")
    dst = tmp_path / "draft_sampling_verification_head_b200" / "csrc"
    shutil.copytree(src, dst)
    root = str(tmp_path)
    h0 = {n: bench.kernel_hash(n, root) for n in bench.PROFILED_SOURCES}
    assert h0 == {n: bench.kernel_hash(n) for n in bench.PROFILED_SOURCES}
    cyc = dst / "cycle_tc.cu"
    cyc.write_text(cyc.read_text() + "\n// a comment only\n/* and a block\n comment */\n")
    assert bench.kernel_hash("k_cycle_tc_c3", root) == h0["k_cycle_tc_c3"]
    cyc.write_text(cyc.read_text() + "\nnamespace { constexpr int kProbe = 1; }\n")
    assert bench.kernel_hash("k_cycle_tc_c3", root) != h0["k_cycle_tc_c3"]
    assert bench.kernel_hash("k_verify_ee_c3", root) == h0["k_verify_ee_c3"]  # another kernel's file
    hdr = dst / "common.cuh"
    hdr.write_text(hdr.read_text() + "\nnamespace { constexpr int kProbe2 = 2; }\n")
    assert bench.kernel_hash("k_verify_ee_c3", root) != h0["k_verify_ee_c3"]  # a shared header
