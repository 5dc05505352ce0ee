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


class _FakeEvent:
    def __init__(self, enable_timing=False):
        pass

    def record(self, stream=None):
        pass

    def elapsed_time(self, other):
        return 2.0


class _FakeLibrary:
    """Every entry point of the binding does nothing and counts the call."""

    def __init__(self):
        self.calls = {}

    def __getattr__(self, name):
        if not name.startswith("fp8bw_"):
            raise AttributeError(name)

        def call(*args, **kwargs):
            self.calls[name] = self.calls.get(name, 0) + 1
        return call


class _FakeLinear:
    def __init__(self, kind, k, n):
        import torch
        self.kind, self.k, self.n = kind, k, n
        for attr in ("x", "dy", "dw", "w", "qx", "sx", "qw", "sw", "qw_t", "qdy", "sdy",
                     "qdy_t", "sdy_t", "qx_t", "sx_t", "y", "dx"):
            setattr(self, attr, torch.zeros(1))

    def weight_bytes(self):
        return 1e6

    def ops(self, o, stream, pow2=False):
        return [("quant_rowcol", 1e6, lambda: None),
                ("gemm_block_scaled", 1e9, lambda: None)]

    def wgrad_job(self):
        return (self.qdy_t, self.sdy_t, self.qx_t, self.sx_t, None)


def test_next_rows_host_logic_with_stubbed_device(monkeypatch):
    """time_next_rows end to end on the CPU: CUDA events and streams stubbed,
    every library call a no-op; checks the rows, their units and texts."""
    import contextlib
    import torch
    monkeypatch.setattr(torch.cuda, "Event", _FakeEvent)
    monkeypatch.setattr(torch.cuda, "stream", lambda s: contextlib.nullcontext())
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a: None)
    monkeypatch.setattr(bench, "TOKENS", 256)
    lib = _FakeLibrary()
    bufs = [_FakeLinear("gate_up", 128, 256), _FakeLinear("down", 256, 128)]
    out = bench.time_next_rows(lib, bufs, None, 3, 5)
    assert set(out) == {"wgrad_f32_accumulate", "gemm_fused_rowwise_quant",
                        "gemm_fused_rowcol_quant", "pow2_step", "configs"}
    # the MLP configurations' kernels, one at a time (no QKV linear here)
    assert set(out["configs"]["rows"]) == {
        k + "_" + r for k in ("gate_up", "down")
        for r in ("quant_x_rowcol", "fprop", "quant_dy_rowcol", "dgrad", "wgrad")}
    assert "gate/up and down linears" in out["wgrad_f32_accumulate"]["what"]
    assert "gate/up and down linears" in out["gemm_fused_rowwise_quant"]["what"]
    assert "gate/up and down linears" in out["gemm_fused_rowcol_quant"]["what"]
    assert lib.calls["fp8bw_gemm_fprop_quant_rowcol"] == \
        lib.calls["fp8bw_gemm_dgrad_quant_rowcol"]
    assert ("%d-layer" % bench.LAYERS) in out["pow2_step"]["what"]
    assert out["wgrad_f32_accumulate"]["launches"] == 5
    assert lib.calls["fp8bw_gemm_wgrad_f32_batch"] == 3 + 5
    # the power-of-two step: one batched wgrad per layer
    assert lib.calls["fp8bw_gemm_wgrad_batch"] == 3 * bench.LAYERS + 3 * bench.LAYERS
    # fprop runs in the row-wise and the row + column comparison alike, and
    # in the configurations' timing (2 warm-up + 5 timed calls per linear)
    assert 2 * lib.calls["fp8bw_gemm_fprop_quant"] + 2 * (2 + 5) == \
        lib.calls["fp8bw_gemm_fprop"]
    assert set(out["pow2_step"]["breakdown"]) == {
        "quant_weight_block", "quant_rowcol", "gemm_block_scaled",
        "gemm_vector_scaled"}
    assert all(v["unit"] == "TFLOP/s" for k, v in out.items() if k != "configs")
    assert all(r["unit"] == ("TFLOP/s" if k.endswith(("fprop", "dgrad", "wgrad")) else "GB/s")
               for k, r in out["configs"]["rows"].items())
