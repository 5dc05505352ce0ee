"""Host-side pieces of bench.py: the nvidia-smi clock summary (only samples
inside the timed window, throttle reasons that were active) and the rule
that ncu traffic is reported only for the kernel sources it was taken on."""
import datetime

import bench


def _line(t, mhz, reasons=()):
    ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    flags = ["Active" if n in reasons else "Not Active" for n in names]
    return ", ".join([ts, "0", str(mhz), "1965", "950.0", "0x4"] + flags)


def test_clock_summary_keeps_the_timed_window():
    t0 = 1_800_000_000.0
    out = "\n".join([_line(t0 - 0.5, 1965)] +                        # before: idle
                    [_line(t0 + 0.2 * i, 1650 + i, ("sw_power_cap",)) for i in range(5)] +
                    [_line(t0 + 2.0, 1965, ("hw_slowdown",))])        # after
    s = bench.ClockSampler.summarise(out, (t0, t0 + 1.0))
    assert s["samples"] == 5 and s["sm_mhz"] == 1652 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]
    everything = bench.ClockSampler.summarise(out)
    assert everything["samples"] == 7 and "hw_slowdown" in everything["reasons"]
    # no sample inside the window: all samples are used
    assert bench.ClockSampler.summarise(out, (t0 + 10, t0 + 11))["samples"] == 7
    assert bench.ClockSampler.summarise("garbage\n") is None


def test_ncu_traffic_only_for_the_recorded_sources(monkeypatch):
    k = "gemm_block_scaled"
    monkeypatch.setattr(bench, "KERNEL_FINGERPRINT", bench.kernel_fingerprint())
    assert bench.ncu_traffic(k) == bench.NCU_TRAFFIC_PER_LAUNCH[k]
    monkeypatch.setattr(bench, "KERNEL_FINGERPRINT", "0" * 16)
    assert bench.ncu_traffic(k) is None


def test_clock_summary_without_timestamps():
    line = "n/a, 0, 1700, 1965, 900.0, 0x0, Not Active, Not Active, Not Active, Not Active"
    s = bench.ClockSampler.summarise("\n".join([line] * 3), (0.0, 1.0))
    assert s["samples"] == 3 and s["sm_mhz"] == 1700 and s["reasons"] == []


def test_linear_names():
    assert bench.linear_names(["qkv", "o", "gate_up", "down"]) == \
        "QKV, O, gate/up and down"
    assert bench.linear_names(["gate_up"]) == "gate/up"
    assert bench.linear_names(["o", "down"]) == "O and down"
