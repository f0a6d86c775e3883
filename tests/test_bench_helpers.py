"""Host logic of bench.py's measurement protocol (CPU only): the statistics of
the timing samples, the clock samples matched to their time windows, the
launch-share record read from profiles/, and the config both arms report."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_sample_stats_median_and_fractions():
    per = [41.0, 40.0, 42.0, 41.5, 40.5, 41.2, 40.8, 41.1, 40.9, 41.3]
    st = bench.sample_stats(per, 6000, 268435456, 6537.3)
    assert st["samples"] == 10 and st["calls_per_sample"] == 6000
    assert st["us_per_call_median"] == pytest.approx(41.05)
    assert st["us_per_call_min"] == 40.0 and st["us_per_call_max"] == 42.0
    gbs = 268435456 / 41.05 / 1e3
    assert st["GB/s"] == pytest.approx(gbs, abs=0.1)
    assert st["frac_measured"] == pytest.approx(gbs / 6537.3, abs=1e-4)
    assert st["frac_spec"] == pytest.approx(gbs / 8000.0, abs=1e-4)


def test_clock_rows_are_parsed_and_matched_to_windows():
    line = ("2026/12/02 17:35:01.250, 1800, 1965, 900.5, 100, Active, Not Active, Not Active, "
            "Not Active, Active")
    r = bench.ClockSampler._parse(line)
    assert r["sm"] == 1800.0 and r["max"] == 1965.0 and r["reasons"] == ["sw_power_cap"]
    assert bench.ClockSampler._parse("garbage") is None
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.rows = [{"t": t, "sm": sm, "max": 1965.0, "power": 500.0, "util": 100.0, "reasons": rs}
              for t, sm, rs in ((1.0, 1965.0, []), (2.0, 1700.0, ["sw_power_cap"]),
                                (3.0, 1750.0, []), (9.0, 1000.0, ["hw_slowdown"]))]
    inside = s.within([(1.5, 3.5)])
    assert inside["samples"] == 2 and inside["sm_mhz"] == 1725.0
    assert inside["reasons"] == ["sw_power_cap"]
    assert s.within([(4.0, 5.0)]) == {"samples": 0}


def test_kernel_times_from_launch_shares():
    shares = {"split_share": 0.9208, "combine_share": 0.0792, "split_us": 40.264,
              "combine_us": 3.462}
    kt = bench.kernel_times(shares, 40.335, 268435456, 6537.3)
    assert kt["split_us"] == pytest.approx(0.9208 * 40.335, abs=1e-3)
    assert kt["split_GB/s"] == pytest.approx(268435456 / (0.9208 * 40.335) / 1e3, abs=0.1)
    assert bench.kernel_times(None, 40.0, 1, 1.0) is None


def test_launch_share_record_matches_the_committed_device_code():
    """profiles/ncu_traffic.json names the device code it was captured on; the
    bench uses it only while the code still hashes to that value."""
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        rec = json.load(f)
    assert rec["source_hash"] == bench.kernel_source_hash()
    e = bench.ncu_launch_shares("codellama34b-gqa8-L65536", 16)
    assert e is not None and abs(e["split_share"] + e["combine_share"] - 1.0) < 1e-3
    assert bench.ncu_launch_shares("codellama34b-gqa8-L65536", 17) is None
    assert bench.ncu_traffic("codellama34b-gqa8-L65536", 16) >= 268435456


def test_both_arms_report_the_same_config():
    from split_kv_decode_attn_b200 import workloads as wl
    w = wl.config(1)
    ours = bench.workload_config(w, 8, 8, 3, 126 * 1024 * 1024, 1)
    assert ours["num_splits"] == 8 and ours["kv_bytes_per_call"] == w.kv_bytes()
    ref = bench.reference_config(w, 1)
    assert set(ref) == set(ours)
    for key in ("workload", "B", "Hq", "Hkv", "D", "max_len", "block_size", "kv_bytes_per_call",
                "parallelism"):
        assert ref[key] == ours[key]
