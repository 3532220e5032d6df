"""Host logic of the benchmark line on CPU: the clock record parsed from nvidia-smi's CSV
(median SM clock under load, maximum clock, throttle reasons that reject a run), and the
ncu traffic figure, reported only for the attention kernel source it was taken on."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _sampler_with(lines):
    s = bench.ClockSampler(0)
    s.out = "\n".join(lines) + "\n"
    return s


# index, clocks.sm, clocks.max.sm, power.draw, reasons.active, hw_slowdown,
# hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap (the query's field order)
def _row(sm, mx=1965, hw="Not Active", hwt="Not Active", swt="Not Active", cap="Not Active"):
    return f"0, {sm}, {mx}, 900.0, 0x0000000000000000, {hw}, {hwt}, {swt}, {cap}"


def test_clock_summary_median_max_and_power_cap():
    s = _sampler_with([_row(1965), _row(1800, cap="Active"), _row(1900), _row(1700, cap="Active"),
                       _row(1965)])
    got = s.summary()
    assert got["sm_mhz"] == 1900.0
    assert got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["sw_power_cap"]
    assert got["samples"] == 5


@pytest.mark.parametrize("field,name", [("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                                        ("swt", "sw_thermal_slowdown")])
def test_clock_summary_reports_every_rejecting_reason(field, name):
    s = _sampler_with([_row(1965), _row(1500, **{field: "Active"})])
    assert name in s.summary()["reasons"]


def test_clock_summary_without_samples_says_so():
    s = _sampler_with([])
    got = s.summary()
    assert got["sm_mhz"] is None and got["reasons"] == ["unsampled"]
    # malformed lines (an nvidia-smi error message) are not samples
    assert _sampler_with(["No devices were found"]).summary()["reasons"] == ["unsampled"]


def test_traffic_only_for_the_kernel_source_it_was_measured_on():
    sha = bench.NCU_ATTN_TRAFFIC["kernel_source_sha"]
    assert bench._attn_traffic(sha) == pytest.approx(bench.NCU_ATTN_TRAFFIC["bytes_per_launch"])
    assert bench._attn_traffic("0" * 16) is None


def test_kernel_source_sha_covers_the_attention_sources():
    sha = bench.kernel_source_sha()
    assert len(sha) == 16 and int(sha, 16) >= 0
    assert sha == bench.kernel_source_sha()  # a pure function of the two files
