"""Host-side logic of bench.py that needs no GPU: the clock sampler keeps only
the nvidia-smi samples taken inside the timed windows, and reports the
throttle reasons seen there."""
import datetime
import os
import sys
import tempfile
import time

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


class _Done:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        pass


def _sampler_with(lines, windows):
    c = bench.ClockSampler(0)
    fd, c.path = tempfile.mkstemp(suffix=".csv")
    os.close(fd)
    with open(c.path, "w") as f:
        f.write("\n".join(lines) + "\n")
    c.proc = _Done()
    c.windows = windows
    return c


def _line(t, mhz, power_cap):
    ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    cap = "Active" if power_cap else "Not Active"
    return f"{ts}, 0, {mhz}, 1965, 950.0, Not Active, Not Active, Not Active, {cap}"


def test_clock_sampler_keeps_only_the_timed_windows():
    t0 = time.time()
    # 20 samples 50 ms apart; the warm-up ones run at 1800 MHz, the timed
    # ones at 1300-1309 MHz under the power cap, the ones after at 600 MHz
    lines = [_line(t0 + 0.05 * k, 1800, False) for k in range(5)]
    lines += [_line(t0 + 0.05 * k, 1300 + k - 5, True) for k in range(5, 15)]
    lines += [_line(t0 + 0.05 * k, 600, False) for k in range(15, 20)]
    lines.insert(3, "garbage, line")
    c = _sampler_with(lines, [(t0 + 0.24, t0 + 0.71)])
    r = c.stop()
    assert r["samples"] == 10
    assert r["sm_mhz"] == 1304.5
    assert r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]
    assert not os.path.exists(c.path)


def test_clock_sampler_several_windows_and_none_inside():
    t0 = time.time()
    lines = [_line(t0 + 0.1 * k, 1400 + k, False) for k in range(10)]
    r = _sampler_with(lines, [(t0 - 0.01, t0 + 0.11), (t0 + 0.69, t0 + 0.81)]).stop()
    assert r["samples"] == 4 and r["reasons"] == []
    assert r["sm_mhz"] == (1401 + 1407) / 2
    assert _sampler_with(lines, [(t0 + 5.0, t0 + 6.0)]).stop() is None
