"""Host-side pieces of the bench line, on the CPU: the `roofline` object (the HBM form for
the rank-space kernels, the tensor-pipe form for the keys-before-RoPE kernel) from fixed
timings, and the clock record built from nvidia-smi samples."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402

PEAKS = {"hbm_gbs": 6538.0, "bf16_tflops": 1642.8, "bf16_tflops_sustained": 1399.6}


def test_hbm_roofline():
    r = bench.roofline_entry("decode_tc", 67108864, 0.0, 0.0231, PEAKS, "measured",
                             {"bytes_per_launch": 69212160})
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(67108864 / 23.1e-6 / 1e9, abs=0.1)
    assert r["frac"] == pytest.approx(r["achieved"] / 6538.0, abs=1e-4)
    assert r["peak"] == 6538.0 and r["traffic"] == 69212160 and r["kernel_us"] == 23.1


def test_tensor_roofline_for_keys_before_rope():
    flops = 4.0587e12
    r = bench.roofline_entry("decode_tc_i4_rope", 4.8234e9, flops, 17.09991, PEAKS, "measured", None)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(flops / 17.09991e-3 / 1e12, abs=0.1)
    assert r["frac"] == pytest.approx(r["achieved"] / 1399.6, abs=1e-4)
    assert r["hbm_gbs"] == pytest.approx(4.8234e9 / 17.09991e-3 / 1e9, abs=0.1)
    assert r["traffic"] is None and r["flops_per_step"] == flops


def test_fallback_peaks():
    r = bench.roofline_entry("decode_tc", 1e9, 0.0, 1.0, {}, "fallback", None)
    assert r["peak"] == bench.FALLBACK_HBM_GBS
    r = bench.roofline_entry("decode_tc_i4_rope", 1e9, 1e12, 1.0, {}, "fallback", None)
    assert r["peak"] == bench.FALLBACK_TFLOPS_SUSTAINED


def test_clock_summary_filters_gpu_and_reports_reasons():
    class FakeProc:
        stdout = [
            "GPU-aaa, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active\n",
            "GPU-bbb, 300, 1965, 90.0, 0x0, Active, Not Active, Not Active, Not Active\n",
            "GPU-aaa, 1890, 1965, 998.0, 0x4, Not Active, Not Active, Not Active, Active\n",
            "GPU-aaa, 1950, 1965, 980.0, 0x0, Not Active, Not Active, Not Active, Not Active\n",
            "malformed line\n",
        ]
    cs = bench.ClockSampler("GPU-aaa")
    cs.proc = FakeProc()
    cs._read()
    s = cs.summary()
    assert s["samples"] == 3                       # the other GPU's row and the malformed one are dropped
    assert s["sm_mhz"] == 1950.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]        # another GPU's hw_slowdown is not ours


def test_clock_summary_without_samples():
    s = bench.ClockSampler("GPU-aaa").summary()
    assert s["samples"] == 0 and s["reasons"] == ["unsampled"]


def test_percentile_matches_numpy_linear():
    import numpy as np
    rng = np.random.default_rng(0)
    for n in (1, 2, 5, 20, 51):
        v = list(rng.standard_normal(n))
        for q in (0, 10, 50, 90, 100):
            assert abs(bench.percentile(v, q) - float(np.percentile(v, q))) < 1e-12
