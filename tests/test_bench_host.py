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
