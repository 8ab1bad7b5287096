"""The benchmark's clock record (the nvidia-smi samples taken during the timed region), parsed
from fake sample lines: the GPU's own rows only, the median SM clock under load, the throttle
reasons seen, the power maximum.  CPU only; nothing is launched."""
import bench


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _sampler(lines, bus_id=None, index=None):
    s = bench.ClockSampler(bus_id=bus_id, index=index)
    s.proc = _FakeProc()
    s.out = list(lines)
    return s


def _line(idx, bus, sm, smax, power, hw="Not Active", hwt="Not Active", swt="Not Active", cap="Not Active"):
    return ", ".join([str(idx), bus, str(sm), str(smax), str(power), hw, hwt, swt, cap])


def test_own_rows_median_under_load_and_reasons():
    lines = [
        _line(0, "00000000:1B:00.0", 1965, 1965, 700.5),
        _line(1, "00000000:43:00.0", 800, 1965, 200.0, hw="Active"),  # another GPU: ignored
        _line(0, "00000000:1B:00.0", 1950, 1965, 720.0, cap="Active"),
        _line(0, "00000000:1B:00.0", 345, 1965, 150.0),                # idle sample: not under load
        _line(0, "00000000:1B:00.0", 1965, 1965, 690.0),
        "garbled line",
    ]
    r = _sampler(lines, bus_id="00000000:1B:00.0").stop()
    assert r["samples"] == 4 and r["sm_max_mhz"] == 1965.0
    assert r["sm_mhz"] == 1965.0  # median of the three loaded samples
    assert r["reasons"] == ["sw_power_cap"] and r["power_w_max"] == 720.0
    r = _sampler(lines, index=1).stop()
    assert r["samples"] == 1 and r["reasons"] == ["hw_slowdown"]


def test_power_not_reported_and_no_samples():
    lines = [_line(0, "00000000:1B:00.0", 1965, 1965, "[N/A]")]
    r = _sampler(lines, index=0).stop()
    assert r["samples"] == 1 and r["power_w_max"] is None and r["reasons"] == []
    r = _sampler([], index=0).stop()
    assert r["samples"] == 0 and r["reasons"] == ["no samples"]
    s = bench.ClockSampler(index=0)
    assert s.stop()["reasons"] == ["nvidia-smi unavailable"]
