"""bench.py's clock summary keeps only the samples of the timed region."""

import datetime
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402

NA = "Not Active"


def _row(ts, sm, reasons=(NA, NA, NA, NA)):
    return ", ".join([ts.strftime("%Y/%m/%d %H:%M:%S.%f")[:-3], "0", str(sm), "1965", "700.5",
                      "0x0000000000000000", *reasons])


def test_only_samples_inside_the_timed_region_count():
    t = datetime.datetime(2026, 12, 2, 22, 0, 0)
    ms = lambda x: t + datetime.timedelta(milliseconds=x)
    text = "\n".join([
        _row(ms(0), 1965), _row(ms(100), 1965),                       # before: idle
        _row(ms(200), 1500), _row(ms(300), 1520), _row(ms(400), 1480,
                                                        (NA, NA, NA, "Active")),
        _row(ms(500), 1965, ("Active", NA, NA, NA)),                   # after the region
    ])
    s = bench.summarise_clocks(text, ms(150), ms(450))
    assert s["samples"] == 3 and s["sm_mhz"] == 1500 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"] and s["window"] == "timed region"


def test_short_region_falls_back_to_the_nearest_samples():
    t = datetime.datetime(2026, 12, 2, 22, 0, 0)
    ms = lambda x: t + datetime.timedelta(milliseconds=x)
    text = "\n".join([_row(ms(0), 1900), _row(ms(100), 1700), _row(ms(200), 1800)])
    s = bench.summarise_clocks(text, ms(110), ms(130))   # no sample inside
    assert s["window"] == "nearest to the timed region"
    assert s["samples"] == 1 and s["sm_mhz"] == 1700


def test_unparseable_output_gives_none():
    assert bench.summarise_clocks("", None, None) is None
    assert bench.summarise_clocks("garbage\n1,2,3", None, None) is None


def test_nvml_sampler_gives_several_samples_in_a_short_region(monkeypatch):
    """The NVML sampler (here a fake module: no GPU needed) records every few
    ms, so a timed region of tens of ms still holds several samples; the
    reason bits map to the named throttle reasons."""
    import time
    import types
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=1,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByIndex=lambda i: ("h", i),
        nvmlDeviceGetHandleByUUID=lambda u: ("h", u),
        nvmlDeviceGetMaxClockInfo=lambda h, c: 1965,
        nvmlDeviceGetClockInfo=lambda h, c: 1800,
        nvmlDeviceGetPowerUsage=lambda h: 812000,
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: 0x4,   # sw_power_cap
    )
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    c = bench.ClockSampler(0, "GPU-fake", period_s=0.002)
    c.start()
    time.sleep(0.02)
    c.mark()
    time.sleep(0.06)
    c.mark(end=True)
    s = c.stop()
    assert s["samples"] >= 5 and s["window"] == "timed region"
    assert s["sm_mhz"] == 1800 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"] and s["source"].startswith("NVML")
