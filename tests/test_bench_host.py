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
