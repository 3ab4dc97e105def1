"""Host-side pieces of bench.py: algorithmic work accounting and the
recorded-traffic lookup (no GPU)."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from transformer_layer_pre_b200.synthetic import WORKLOADS  # noqa: E402


def test_step_flops_bert_large():
    # 77.07 MFLOP per token fwd+bwd at H1024 F4096 S128: 6*(4H^2+2HF) + 12*S*H
    w = WORKLOADS["bert-large-f16"]
    per_tok = bench.linear_flops_per_token(w.hidden, w.ffn) + bench.attn_flops_per_token(w.seq, w.hidden)
    assert per_tok == 6 * (4 * 1024 ** 2 + 2 * 1024 * 4096) + 12 * 128 * 1024
    assert abs(per_tok * w.tokens / 1e9 - 631.36) < 0.01


def test_recorded_traffic_tracks_kernel_sources(monkeypatch, tmp_path):
    prof = tmp_path / "gemm.txt"
    prof.write_text(f"summary\nTRAFFIC_BYTES_PER_LAUNCH 67381248\nKERNEL_SOURCES_SHA256 {bench.gemm_sources_digest()}\n")
    monkeypatch.setattr(bench, "GEMM_PROFILE", str(prof))
    assert bench.recorded_gemm_traffic(bench.WORKLOAD) == 67381248.0
    assert bench.recorded_gemm_traffic("tiny-f32") is None
    # a changed kernel source invalidates the recorded counters
    monkeypatch.setattr(bench, "gemm_sources_digest", lambda: "0" * 64)
    assert bench.recorded_gemm_traffic(bench.WORKLOAD) is None


def test_clock_sampler_reads_a_fake_nvml_and_only_reads(monkeypatch):
    """The clock record: samples only inside the timed region, from the
    main thread's sample() as well as the thread, throttle reasons decoded
    from the reason mask; every NVML call it makes is a query."""
    import types
    calls = []
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=0,
        nvmlClocksEventReasonHwSlowdown=0x8, nvmlClocksEventReasonHwThermalSlowdown=0x40,
        nvmlClocksEventReasonSwThermalSlowdown=0x20, nvmlClocksEventReasonSwPowerCap=0x4)

    def rec(name, value):
        def f(*a):
            calls.append(name)
            return value
        return f
    fake.nvmlInit = rec("nvmlInit", None)
    fake.nvmlDeviceGetHandleByPciBusId = rec("nvmlDeviceGetHandleByPciBusId", "h")
    fake.nvmlDeviceGetHandleByIndex = rec("nvmlDeviceGetHandleByIndex", "h")
    fake.nvmlDeviceGetMaxClockInfo = rec("nvmlDeviceGetMaxClockInfo", 1965)
    fake.nvmlDeviceGetClockInfo = rec("nvmlDeviceGetClockInfo", 1800)
    fake.nvmlDeviceGetCurrentClocksEventReasons = rec("nvmlDeviceGetCurrentClocksEventReasons", 0x6)
    fake.nvmlClocksEventReasonApplicationsClocksSetting = 0x2
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    with bench.ClockSampler(0, period_s=10.0) as clk:   # the thread wakes too rarely to sample
        clk.sample()                                      # outside the timed region: ignored
        clk.timed = True
        clk.sample()
        clk.sample()
        clk.timed = False
    s = clk.summary()
    assert s["samples"] == 2 and s["sm_mhz"] == 1800 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["applications_clocks_setting", "sw_power_cap"]
    assert all(c == "nvmlInit" or c.startswith("nvmlDeviceGet") for c in calls)
