"""Host-side logic of bench.py that needs no GPU: the nvidia-smi clock
sampler's parsing and the reporting of throttle reasons."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

def test_clock_sampler_parses_and_flags_throttling():
    """bench.Clocks reads `nvidia-smi --query-gpu=... --format=csv,noheader,nounits`
    samples; the median SM clock and every active slowdown reason are reported."""
    sys.path.insert(0, ROOT)
    import bench

    class FakeProc:
        def __init__(self, out):
            self.out = out

        def terminate(self):
            pass

        def communicate(self, timeout=None):
            return self.out, ""

    rows = ["0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
            "0, 1950, 1965, 980.5, 0x4, Not Active, Not Active, Not Active, Active",
            "0, 1965, 1965, 990.0, 0x4, Not Active, Active, Not Active, Active",
            "garbage line"]
    c = bench.Clocks.__new__(bench.Clocks)
    c.proc = FakeProc("\n".join(rows))
    d = c.stop()
    assert d["sm_mhz"] == 1965.0 and d["sm_max_mhz"] == 1965.0 and d["samples"] == 3
    assert d["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    c.proc = None
    assert c.stop()["sm_mhz"] is None
