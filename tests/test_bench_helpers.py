"""Host arithmetic of bench.py's secondary measurements (no GPU): miss rates by
phase from a cache event trace, the prefill GEMM's roofline, and the share of
compute hidden under the prefetch copies."""
import numpy as np
import pytest

import bench
import synth
from oracle.lru import HIT, MISS, LRUCache


def test_event_kinds_match_the_abi():
    assert (bench.EV_HIT, bench.EV_MISS) == (HIT, MISS)


def test_miss_phases_agree_with_a_per_token_count():
    # a small decode run over an LRU with a shrink and a restore; the trace's
    # lookups are split per token and counted directly
    layers, tokens, E, k = 3, 30, 32, 4
    sets = np.stack([synth.zipf_trace(5, l, tokens, E, k, 1.0, 0.5) for l in range(layers)], axis=1)
    lru, ev, per_token_misses = LRUCache(40), [], []
    for p in range(tokens):
        if p == 10:
            ev += lru.resize(20)
        if p == 20:
            ev += lru.resize(40)
        m = 0
        for l in range(layers):
            step = lru.step(l, sets[p, l])
            m += sum(1 for e in step if e[0] == MISS)
            ev += step
        per_token_misses.append(m)
    per = layers * k
    got = bench.miss_phases(ev, per, [("cold", (0, 1)), ("a", (1, 10)), ("b", (10, 20)), ("c", (20, 30))])
    assert got["cold"] == 1.0                       # an empty cache misses every lookup
    for name, (a, b) in [("a", (1, 10)), ("b", (10, 20)), ("c", (20, 30))]:
        assert got[name] == pytest.approx(sum(per_token_misses[a:b]) / ((b - a) * per), abs=0)


def test_miss_phases_refuse_a_trace_of_another_length():
    ev = [(HIT, 0, 1, 0, -1)] * 7
    assert bench.miss_phases(ev, 4, [("x", (0, 2))]) is None


def test_prefill_roofline_of_the_dsv4_class_layer():
    H, I, E, k, T = 4096, 2048, 256, 6, 4096
    flops = 2.0 * T * k * 3 * H * I
    wbytes = E * 3 * H * I * 17 // 32                # codes + UE8M0 scales of every expert
    r = bench.prefill_roofline(flops, wbytes, 6544.7, 1064.0)
    # ~96 tokens per expert: 2 x 96 FLOP per weight over 17/32 byte per weight
    assert r["flop_per_weight_byte"] == pytest.approx(2 * T * k / E * 32 / 17, rel=1e-12)
    assert r["bound"] == "hbm"
    assert r["roofline_tflops"] == pytest.approx(6544.7 * r["flop_per_weight_byte"] / 1e3)
    assert r["frac_of_roofline"] == pytest.approx(1064.0 / r["roofline_tflops"])
    # enough tokens per expert moves the ridge past the tensor peak
    big = bench.prefill_roofline(flops * 64, wbytes, 6544.7, 1.0)
    assert big["bound"] == "tensor" and big["roofline_tflops"] == bench.FP4_DENSE_TFLOPS_NOMINAL


def test_overlap_fraction_limits():
    n, copy, comp = 3, 60.0, 1.5
    serial = n * (copy + comp)
    pipelined = n * copy + comp                      # only the last compute is exposed
    assert bench.overlap_fraction(n * copy, n * comp, serial, (n - 1) * comp) == 0.0
    assert bench.overlap_fraction(n * copy, n * comp, pipelined, (n - 1) * comp) == 1.0
    assert bench.overlap_fraction(n * copy, n * comp, pipelined + comp / 2, (n - 1) * comp) == pytest.approx(0.75)
    assert bench.overlap_fraction(n * copy, n * comp, 1.0, (n - 1) * comp) == 1.0      # clamped
    assert bench.overlap_fraction(copy, comp, copy + comp, 0.0) is None


def test_clock_reason_bits_match_nvml():
    import pynvml
    names = {"gpu_idle": "GpuIdle", "applications_clocks_setting": "ApplicationsClocksSetting",
             "sw_power_cap": "SwPowerCap", "hw_slowdown": "HwSlowdown", "sw_thermal_slowdown": "SwThermalSlowdown",
             "hw_thermal_slowdown": "HwThermalSlowdown", "hw_power_brake_slowdown": "HwPowerBrakeSlowdown",
             "display_clock_setting": "DisplayClockSetting"}
    for bit, name in bench.ClockSampler.REASONS.items():
        assert getattr(pynvml, "nvmlClocksEventReason" + names[name]) == bit


class FakeNvml:
    """Stands in for pynvml during a timed region: SM clocks and the
    clock-event reason bits it reports, one sample per poll."""
    NVML_CLOCK_SM = 1

    def __init__(self, clocks, reasons):
        self.clocks, self.reasons, self.i = clocks, reasons, 0

    def nvmlDeviceGetClockInfo(self, h, which):
        return self.clocks[min(self.i, len(self.clocks) - 1)]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        v = self.reasons[min(self.i, len(self.reasons) - 1)]
        self.i += 1
        return v


def test_clock_sampler_reports_median_and_every_reason_seen():
    import time
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.samples, s.reasons, s.max_mhz, s.h = [], 0, 1965, None
    s._stop = bench.threading.Event()
    s.nv = FakeNvml([1965, 1950, 1965, 1300, 1965], [0x1, 0x4, 0x0, 0x0, 0x20])
    with s:
        time.sleep(0.2)
    out = s.summary()
    assert out["sm_max_mhz"] == 1965 and out["samples"] == len(s.samples) >= 5
    assert out["sm_mhz"] == 1965                                  # median, not the dip
    assert out["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]   # idle is not a throttle reason


def test_clock_sampler_without_nvml_says_so():
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.samples, s.reasons, s.max_mhz, s.nv = [], 0, None, None
    s._stop = bench.threading.Event()
    with s:
        pass
    assert s.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}


def test_stack_launch_counts_follow_the_runtime_paths(monkeypatch):
    """Launches of one stacked pass, as bench.py counts them for its
    gpu_launches claim: the routing kernel and one dataflow launch for up to
    two tokens, both per wave of two for three or four, the routing kernel
    and the counter kernel with FT_STACK_COUNTERS, and the routing kernel plus
    two kernels per layer layerwise (the 35B-class 40-layer stack)."""
    import bench
    monkeypatch.setattr(bench, "L", 40)
    assert [bench.stack_launches(T) for T in (1, 2, 3, 4)] == [2, 2, 4, 4]
    assert bench.stack_launches(4, counters=True) == 2
    assert bench.stack_launches(1, layerwise=True) == 81
    assert "waves of two" in bench.decode_kernel_name(4) and "waves" not in bench.decode_kernel_name(2)
    assert "counter" in bench.decode_kernel_name(8)
