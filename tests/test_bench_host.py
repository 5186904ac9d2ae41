"""Host logic of bench.py that needs no GPU: the clock summary attached to every JSON line
(window filtering, median, throttle reasons from NVML samples or nvidia-smi lines) and the
algorithmic FLOP/byte model behind the roofline."""
import numpy as np
import pytest

import bench
from mixture_experts_routed_histogram_b200 import inputs as I


def _sampler(samples=(), lines=(), window=None):
    c = bench.ClockSampler(0)
    c.samples = list(samples)
    c.lines = list(lines)
    c.window = window
    return c


def test_clock_summary_nvml_window_median_and_reasons():
    s = [(0.5, 1965.0, 1965.0, []),                       # before the window: ignored
         (1.0, 1800.0, 1965.0, ["sw_power_cap"]),
         (1.1, 1700.0, 1965.0, []),
         (1.2, 1500.0, 1965.0, ["sw_power_cap"]),
         (3.0, 900.0, 1965.0, ["hw_slowdown"])]           # after the window: ignored
    got = _sampler(samples=s, window=(0.9, 1.25)).summary()
    assert got["sm_mhz"] == 1700.0 and got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["sw_power_cap"] and got["samples"] == 3
    assert got["source"].startswith("nvml")


def test_clock_summary_falls_back_to_last_samples_when_window_is_empty():
    s = [(0.1, 1965.0, 1965.0, []), (0.2, 1900.0, 1965.0, []), (0.3, 1300.0, 1965.0, [])]
    got = _sampler(samples=s, window=(5.0, 6.0)).summary()
    assert got["samples"] == 2 and got["sm_mhz"] == 1600.0


def test_clock_summary_nvidia_smi_lines():
    row = "0, {sm}, 1965, 900.0, 0x4, {hw}, Not Active, Not Active, {pc}"
    lines = [(1.0, row.format(sm=1410, hw="Not Active", pc="Active")),
             (1.1, row.format(sm=1395, hw="Not Active", pc="Active")),
             (1.2, "garbage"),
             (1.3, row.format(sm=1500, hw="Active", pc="Not Active"))]
    got = _sampler(lines=lines, window=(0.9, 1.2)).summary()
    assert got["source"] == "nvidia-smi" and got["samples"] == 3
    assert got["sm_mhz"] == 1410.0
    assert got["reasons"] == ["hw_slowdown", "sw_power_cap"]


def test_clock_summary_without_samples_is_none():
    assert _sampler().summary() is None


@pytest.mark.parametrize("name", ["qwen3_30b_a3b", "nemotron_relu2", "qwen3_30b_a3b_shared1",
                                  "fp8_mxfp4", "decode"])
def test_algorithmic_model_matches_the_headline_flops(name):
    wl = I.WORKLOADS[name]
    counts = np.full(wl.E_all, max(1, wl.R // wl.E_all))
    f, b, b_alg, ne = bench.algorithmic(wl, counts)
    assert f["gemm1_swiglu"] + f["gemm2"] == pytest.approx(wl.flops())
    assert b["route_permute"] == b["route"] + b["permute"]
    assert ne == wl.E_all
    # the weights of every busy expert are read at least once per pass
    wbytes = (0.5 + 1.0 / 32) if wl.dtype == "fp8_mxfp4" else 2.0
    assert b_alg >= (wl.gemm1_rows + wl.I) * wl.E_all * wl.H * wbytes


def test_algorithmic_counts_only_busy_experts():
    wl = I.WORKLOADS["decode"].with_T(1)
    counts = np.zeros(wl.E_all, dtype=np.int64)
    counts[[2, 5]] = 1
    _, b, _, ne = bench.algorithmic(wl, counts)
    assert ne == 2
    assert b["gemm2"] == pytest.approx(2 * wl.H * wl.I * 2.0 + wl.R * wl.I * 2 + wl.R * wl.H * 2)
