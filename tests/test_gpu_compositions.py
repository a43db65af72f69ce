"""Whole-block and tower wiring on the GPU, against closed forms (bit-exact).

A block whose four linear weights are zero quantises them to zero codes and zero
scales, so each GEMM returns exactly bf16(bias + residual): the block output is
bf16(bf16(x + b_proj) + b_fc2) whatever the attention computes.  That checks the
residual connections, the bias placement and the in-place update of x at full
size with no tolerance, and, in a tower of such blocks, that the mergers receive
the states after blocks 8, 16, 24 and 27.
"""
import numpy as np
import pytest
import torch

from oracle import numerics as nm
from oracle import vit as ov
from quantized_vit_encoder_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _zero_linear_params(seed):
    p = wl.block_params(seed)
    for name in ("qkv", "proj", "fc1", "fc2"):
        p[name + "_w"] = torch.zeros_like(p[name + "_w"])
    return p


def _f64(t):
    return t.detach().float().cpu().double().numpy()


@pytest.mark.parametrize("grids", [[(46, 136)], [(36, 27), (16, 16)]], ids=["46x136", "packed"])
def test_block_with_zero_linears_is_its_residual_adds(lib, grids):
    from quantized_vit_encoder_b200 import vitq
    p = _zero_linear_params(31)
    blk = vitq.DeviceBlock(p)
    pos, cu = vitq.positions(grids)
    cs = vitq.rope_table(pos)
    n = pos.shape[0]
    x = wl.random_bf16((n, 1152), 32, 1.0)
    ws = vitq.workspace(vitq.block_workspace_bytes(n))
    got = vitq.block_forward_(blk, x.cuda(), cu, max(h * w for h, w in grids), cs, ws)
    torch.cuda.synchronize()
    assert vitq.device_error() == 0
    x1 = nm.bf16_round(_f64(x) + _f64(p["proj_b"]))
    want = nm.bf16_round(x1 + _f64(p["fc2_b"]))
    assert np.array_equal(_f64(got), want)


def test_tower_of_zero_linear_blocks_taps_after_blocks_8_16_24_27(lib):
    from quantized_vit_encoder_b200 import vitq
    grids = [(16, 16)]
    n = 256
    params = [_zero_linear_params(300 + b) for b in range(wl.N_BLOCKS)]
    mparams = [wl.merger_params(400 + t) for t in range(4)]
    tower = vitq.DeviceTower([vitq.DeviceBlock(p) for p in params], [vitq.DeviceMerger(m) for m in mparams])
    x = wl.random_bf16((n, 1152), 33, 1.0)
    ws = vitq.workspace(vitq.tower_workspace_bytes(n, 1))
    taps = vitq.tower_forward_(tower, x.cuda(), grids, ws)
    torch.cuda.synchronize()
    assert vitq.device_error() == 0
    states = [_f64(x)]
    for p in params:
        x1 = nm.bf16_round(states[-1] + _f64(p["proj_b"]))
        states.append(nm.bf16_round(x1 + _f64(p["fc2_b"])))
    # each merger is fed the exact state, so only the merger's own tolerance remains
    for t, b in enumerate((8, 16, 24, 27)):
        m = ov.quantize_merger_weights({k: _f64(v) for k, v in mparams[t].items()})
        ref = ov.merger_forward(states[b], m)
        got = _f64(taps[t])
        rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
        assert rel < 1e-2, f"tap {t} (after block {b}): rel-L2 {rel:.3e}"
