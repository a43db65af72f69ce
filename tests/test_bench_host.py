"""Host-side pieces of bench.py: the algorithmic FLOP count and the clock-record summary."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_tower_flops_at_46x136():
    n = 46 * 136
    linears = [(3456, 1152), (1152, 1152), (4304, 1152), (1152, 4304)]          # (out, in) of qkv, proj, fc1, fc2
    gemm = sum(2 * n * o * i for o, i in linears)
    attn = 16 * 2 * (2 * n * n * 72)                                            # QK^T and PV per head
    m = n // 4
    merger = 2 * m * 4608 * 4608 + 2 * m * 2048 * 4608
    f = bench.tower_flops([(46, 136)])
    assert f["block_gemm"] == gemm and round(gemm / 1e9, 2) == 190.49
    assert f["block_attn"] == attn and round(attn / 1e9, 2) == 180.35
    assert f["merger"] == merger
    assert f["tower"] == 27 * (gemm + attn) + 4 * merger


def test_packed_images_attend_within_each_image_only():
    grids = [(16, 16), (36, 27)]
    f = bench.tower_flops(grids)
    assert f["block_attn"] == sum(bench.tower_flops([g])["block_attn"] for g in grids)
    assert f["block_gemm"] == sum(bench.tower_flops([g])["block_gemm"] for g in grids)


def test_clock_summary():
    s = bench.ClockSampler(0)
    s.lines = [
        "1965, 1965, 812.3, Not Active, Not Active, Not Active, Not Active",
        "1800, 1965, 1000.1, Not Active, Not Active, Not Active, Active",
        "1890, 1965, 990.0, Not Active, Not Active, Not Active, Active",
        "[N/A], 1965, 990.0, Not Active, Not Active, Not Active, Not Active",   # unreadable sample
        "garbage",
    ]
    d = s.summary()
    assert d["sm_mhz"] == 1890 and d["sm_max_mhz"] == 1965 and d["samples"] == 3
    assert d["reasons"] == ["sw_power_cap"]
    s.lines = ["1200, 1965, 700, Active, Not Active, Active, Not Active"]
    assert s.summary()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert bench.ClockSampler(0).summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def _table():
    # per-kernel event sums as bench.py collects them (two timed steps' worth)
    return {"attention": {"launches": 54, "ms": 15.34, "flops": 54 * 180.35e9, "bytes": 54 * 57.7e6},
            "fp8_block_gemm": {"launches": 232, "ms": 10.48, "flops": 232 * 50e9, "bytes": 232 * 50e6},
            "ln_quant": {"launches": 116, "ms": 3.31, "flops": 0.0, "bytes": 116 * 21.9e6}}


def test_roofline_of_the_dominant_kernel():
    peaks = {"hbm_gbs": 6455.6, "bf16": 1649.5, "bf16_sustained": 1415.6, "source": "measured",
             "fp8": 3300.0, "fp8_sustained": 2900.0, "fp8_source": "measured"}
    r = bench.roofline(_table(), peaks)
    per_launch_s = 15.34e-3 / 54
    assert r["kernel"] == "attention" and r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["achieved"] - 180.35e9 / per_launch_s / 1e12) < 1e-9
    # the burst peak (kernels timed inside a short step), the sustained one as context
    assert r["peak"] == 1649.5 and abs(r["frac"] - r["achieved"] / 1649.5) < 1e-12
    assert r["sustained_peak"] == 1415.6 and abs(r["frac_of_sustained"] - r["achieved"] / 1415.6) < 1e-12
    assert r["nominal_peak"] == 2250.0 and abs(r["frac_of_nominal"] - r["achieved"] / 2250.0) < 1e-12
    assert abs(r["share"] - 15.34 / (15.34 + 10.48 + 3.31)) < 1e-12
    # a GEMM-dominated table takes the measured FP8 peak, an HBM-bound one GB/s
    t = _table()
    t["fp8_block_gemm"]["ms"] = 40.0
    g = bench.roofline(t, peaks)
    assert g["kernel"] == "fp8_block_gemm" and g["peak"] == 3300.0 and g["nominal_peak"] == 4500.0
    assert bench.load_peaks()["fp8"] == 2 * bench.load_peaks()["bf16"]     # before the FP8 measurement
    t["ln_quant"]["ms"] = 100.0
    h = bench.roofline(t, peaks)
    assert h["bound"] == "hbm" and h["unit"] == "GB/s" and h["peak"] == 6455.6
    assert abs(h["achieved"] - 21.9e6 / (100e-3 / 116) / 1e9) < 1e-9


def test_roofline_traffic_only_for_the_profiled_source(monkeypatch):
    """ncu traffic is reported only while the kernel source still hashes to the one profiled."""
    import json
    peaks = bench.load_peaks()
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))["attention"]
    monkeypatch.setattr(bench, "_source_sha", lambda rel: rec["source_sha"])
    assert bench.roofline(_table(), peaks)["traffic"] == rec["bytes_per_launch"]
    monkeypatch.setattr(bench, "_source_sha", lambda rel: "0" * 16)
    assert bench.roofline(_table(), peaks)["traffic"] is None
