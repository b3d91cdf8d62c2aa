"""bench.py's clock record on CPU: the reasons and the median SM clock taken
from nvidia-smi rows, and the record when nvidia-smi is missing."""
import shutil

import pytest

import bench


class _Proc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


class _Thread:
    def join(self, timeout=None):
        pass


def _sampler(rows):
    s = object.__new__(bench.ClockSampler)
    s.rows, s.proc, s.t = rows, _Proc(), _Thread()
    return s


def test_reasons_and_median_clock():
    na, act = "Not Active", "Active"
    rows = [["1965", "1965", "700.1", "0x0", na, na, na, na],
            ["1950", "1965", "980.4", "0x4", na, na, na, act],
            ["1620", "1965", "999.0", "0x4", na, na, na, act],
            ["[N/A]", "1965", "0", "0x0", na, na, na, na]]
    rec = _sampler(rows).stop()
    assert rec["sm_mhz"] == 1950.0          # median of the numeric samples
    assert rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"]
    assert rec["samples"] == 4


def test_throttle_reasons_are_all_reported():
    act, na = "Active", "Not Active"
    rec = _sampler([["1200", "1965", "500", "0x48", act, na, act, na]]).stop()
    assert rec["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


@pytest.mark.skipif(shutil.which("nvidia-smi") is not None, reason="nvidia-smi present")
def test_without_nvidia_smi():
    rec = bench.ClockSampler("0").stop()
    assert rec["sm_mhz"] is None and rec["reasons"] == ["nvidia-smi unavailable"]
