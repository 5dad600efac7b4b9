"""Host-side pieces of bench.py that shape its JSON line: the clock summary
(which decides whether a run is kept), the committed traffic lookup, the
FLOP count of the metric and the roofline denominators.  CPU only."""
import datetime
import os

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _row(t, sm, mx, reasons=("Not Active",) * 4):
    ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    return ", ".join([ts, str(sm), str(mx), "640.12", "0x0000000000000004", *reasons]) + "\n"


def test_clock_summary_median_max_and_reasons():
    t = 1_800_000_000.0
    lines = [_row(t + 0.1, 1965, 1965), _row(t + 0.2, 1920, 1965),
             _row(t + 0.3, 1900, 1965, ("Not Active", "Not Active", "Not Active", "Active")),
             "garbage line\n", _row(t + 0.4, "[N/A]", 1965)]
    s = bench.summarize_clocks(lines)
    assert s["samples"] == 4                       # the malformed line is skipped
    assert s["sm_mhz"] == 1920                     # median of the numeric clocks
    assert s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]        # "Not Active" is not active


def test_clock_summary_keeps_only_the_timed_window():
    t = 1_800_000_000.0
    lines = [_row(t - 5, 1000, 1965, ("Active", "Not Active", "Not Active", "Not Active")),
             _row(t + 1, 1965, 1965), _row(t + 2, 1950, 1965),
             _row(t + 9, 900, 1965, ("Not Active", "Active", "Not Active", "Not Active"))]
    s = bench.summarize_clocks(lines, t, t + 3)
    assert s["samples"] == 2 and s["reasons"] == [] and s["sm_mhz"] == 1957.5
    assert bench.summarize_clocks(lines, t + 20, t + 30) is None
    assert bench.summarize_clocks([]) is None


def test_traffic_is_reported_only_for_the_profiled_source():
    attend = os.path.join(ROOT, "packed_kv_cache_b200", "csrc", "attend.cu")
    other = os.path.join(ROOT, "packed_kv_cache_b200", "csrc", "select.cu")
    got = bench.traffic_for(attend, bench.WORKLOAD)
    # either the committed capture matches this source, or nothing is claimed
    assert got is None or got > 0
    assert bench.traffic_for(other, bench.WORKLOAD) is None
    assert bench.traffic_for(attend, "no such workload") is None


def test_attention_flops_of_the_pages_scale_layer():
    # 4 d_h FLOP per (query, key, head): 12 heads, 6,240 queries, 27,872 keys
    assert bench.attention_flops(1, 12, 6240, 27872) == pytest.approx(1.0686e12, rel=1e-4)
    assert bench.attention_flops(2, 12, 6240, 36608) == 2 * 4 * 12 * 6240 * 36608 * 128


def test_peaks_come_from_the_measured_file_when_present():
    peaks, source = bench.load_peaks()
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        assert source == "measured"
    else:
        assert source == "fallback" and peaks


def test_nvml_reason_bits_decode_to_the_rejecting_names():
    # NVML's clock-event reason bits: sw power cap 0x4, hw slowdown 0x8,
    # sw thermal 0x20, hw thermal 0x40, hw power brake 0x80; idle (0x1) and
    # others are not reported
    assert bench.reason_names(0) == []
    assert bench.reason_names(0x1) == []
    assert bench.reason_names(0x4) == ["sw_power_cap"]
    assert bench.reason_names(0x8 | 0x40) == ["hw_slowdown", "hw_thermal_slowdown"]
    assert bench.reason_names(0x20 | 0x80 | 0x1) == ["hw_power_brake_slowdown", "sw_thermal_slowdown"]


def test_sampled_rows_summarised_inside_the_window():
    rows = [(10.0, 1965.0, 1965.0, []), (10.5, 1900.0, 1965.0, ["sw_power_cap"]), (12.0, 800.0, 1965.0, ["hw_slowdown"])]
    s = bench.summarize_rows(rows, 9.9, 11.0)
    assert s == {"sm_mhz": 1932.5, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 2}
    assert bench.summarize_rows(rows, 20.0, 30.0) is None


def test_timed_window_widened_until_it_holds_samples():
    rows = [(9.0, 1965.0, 1965.0, []), (9.95, 1900.0, 1965.0, ["sw_power_cap"]), (10.06, 1960.0, 1965.0, []),
            (10.2, 1950.0, 1965.0, []), (30.0, 800.0, 1965.0, ["hw_slowdown"])]
    # a 40 ms timed region between two samples: widened 10, 20, 40, 80 ms, then 160 ms each side
    s = bench.summarize_rows_at_least(rows, 10.0, 10.04, n=3)
    assert s["samples"] == 3 and s["pad_s"] == 0.16 and s["window_s"] == 0.36
    assert s["reasons"] == ["sw_power_cap"] and s["sm_mhz"] == 1950.0
    # enough samples inside: left as it is
    s = bench.summarize_rows_at_least(rows, 9.0, 10.2, n=3)
    assert s["samples"] == 4 and s["pad_s"] == 0.0
    # never past max_pad_s: the slow sample 20 s away stays out
    s = bench.summarize_rows_at_least(rows, 10.0, 10.04, n=10, max_pad_s=5.0)
    assert s["samples"] == 4 and s["pad_s"] == 5.0 and "hw_slowdown" not in s["reasons"]
    assert bench.summarize_rows_at_least([], 1.0, 2.0) is None


def test_head_shards_and_roofline_record():
    assert [bench.head_shard(12, 8, r) for r in range(8)] == [(0, 2), (2, 4), (4, 6), (6, 8), (8, 9), (9, 10),
                                                             (10, 11), (11, 12)]
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    r = bench.roofline("k", "hbm", 6e9, 1.0, peaks, "measured")
    assert r["achieved"] == 6000.0 and r["frac"] == 1.0 and r["unit"] == "GB/s"
    r = bench.roofline("k", "tensor", 1.4e12, 1.0, peaks, "measured", sustained=True)
    assert r["achieved"] == 1400.0 and r["frac"] == 1.0 and "sustained" in r["peak_source"]
