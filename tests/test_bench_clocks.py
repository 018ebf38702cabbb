"""The benchmark's summary of the nvidia-smi samples taken during the timed
region: the median SM clock under load (idle samples below half the highest
clock left out), the highest clock the GPU reports, and every throttle
reason seen active in any sample."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

NA = "Not Active"


def _row(sm, hw=NA, hw_th=NA, sw_th=NA, pcap=NA):
    return f"0, {sm}, 1965, 812.40, 0x0000000000000000, {hw}, {hw_th}, {sw_th}, {pcap}\n"


def test_median_under_load_and_no_reasons():
    lines = [_row(345), _row(1965), _row(1950), _row(1965), _row(1965)]
    c = bench.clock_summary(lines)
    assert c["sm_mhz"] == 1965 and c["sm_max_mhz"] == 1965
    assert c["reasons"] == [] and c["samples"] == 5


def test_reasons_are_collected_from_any_sample():
    lines = [_row(1965), _row(1500, pcap="Active"), _row(1200, hw_th="Active"), _row(1965)]
    c = bench.clock_summary(lines)
    assert c["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_unparsable_lines_are_skipped():
    lines = ["garbage\n", "0, [N/A], 1965, 1, 0x0, a, b, c, d\n", _row(1900)]
    c = bench.clock_summary(lines)
    assert c["samples"] == 1 and c["sm_mhz"] == 1900
    assert bench.clock_summary([])["reasons"] == ["no samples"]
