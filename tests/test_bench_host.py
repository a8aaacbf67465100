"""Host logic of bench.py that needs no GPU: the clock sampler keeps only the samples
stamped inside the timed region and reports their median SM clock and every throttle
reason seen there (nvidia-smi's CSV replaced by a written file)."""
import datetime
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _row(t, mhz, active):
    ts = t.strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    reasons = ", ".join("Active" if a else "Not Active" for a in active)
    return f"{ts}, {mhz}, 1965, 700.00, 0x0000000000000000, {reasons}"


def test_clock_sampler_summarises_the_timed_region_only(tmp_path):
    sys.path.insert(0, ROOT)
    import bench
    t = datetime.datetime(2026, 1, 1, 12, 0, 0)
    sec = lambda s: t + datetime.timedelta(seconds=s)
    rows = [
        _row(sec(0.0), 810, (0, 0, 0, 0)),       # before the timed region (idle clock)
        _row(sec(1.0), 1900, (0, 0, 0, 1)),      # inside: power cap active
        _row(sec(1.1), 1965, (0, 0, 0, 0)),
        _row(sec(1.2), 1950, (0, 0, 0, 0)),
        "garbled line",
        _row(sec(3.0), 600, (1, 0, 0, 0)),       # after: hw_slowdown, must not count
    ]
    cs = bench.ClockSampler(0)
    cs.path = str(tmp_path / "clocks.csv")
    with open(cs.path, "w") as f:
        f.write("\n".join(rows) + "\n")

    class Proc:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0
    cs.proc = Proc()
    cs.t0, cs.t1 = sec(0.5), sec(2.0)
    out = cs.stop()
    assert out["samples_in_timed_region"] == 3
    assert out["sm_mhz"] == 1950.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]
    assert not os.path.exists(cs.path)


def test_clock_sampler_without_nvidia_smi_reports_nothing():
    sys.path.insert(0, ROOT)
    import bench
    cs = bench.ClockSampler(0)
    assert cs.stop() is None
