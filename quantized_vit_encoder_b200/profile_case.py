"""Run one stage of the block at the 46x136 (6256-patch) size a few times, for profilers.

    python -m quantized_vit_encoder_b200.profile_case STAGE [--iters N]

STAGE: attention | gemm_qkv | gemm_proj | gemm_fc1 | gemm_fc2 | bf16_qkv | bf16_proj | bf16_fc1 |
       bf16_fc2 | ln_quant | ln_quant_merger | quant_act | gelu_quant | rope | block | tower.
Device memory stays below 0.5 GB except for tower (the 27 blocks' and 4 mergers'
weights, about 1 GB); each iteration is one launch of the stage's kernel (block:
the ten launches of one block; tower: the 288 launches of one tower pass).  The
last iteration runs inside the NVTX range "last_iter", so a profiler can select
exactly its launches (ncu --nvtx --nvtx-include "last_iter/").
"""
from __future__ import annotations

import argparse

import torch

from . import vitq
from . import workloads as wl


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("stage")
    ap.add_argument("--iters", type=int, default=3)
    a = ap.parse_args()
    torch.cuda.set_device(0)
    vitq.load()
    W = wl.WORKLOADS["block_46x136"]
    n = W.n_tokens
    dev = "cuda"
    x = wl.make_input(W).to(dev)
    blk = vitq.DeviceBlock(wl.block_params(wl.block_seed(W, 0)), dev)
    pos, cu = vitq.positions(list(W.grids), dev)
    cs = vitq.rope_table(pos)
    t = blk.t
    if a.stage == "tower":
        blocks = [vitq.DeviceBlock(wl.block_params(wl.block_seed(W, b)), dev) for b in range(wl.N_BLOCKS)]
        mergers = [vitq.DeviceMerger(wl.merger_params(wl.merger_seed(W, m)), dev) for m in range(4)]
        tower = vitq.DeviceTower(blocks, mergers)
        ws = vitq.workspace(vitq.tower_workspace_bytes(n, 1), dev)
        xt = x.clone()
        run = lambda: vitq.tower_forward_(tower, xt.copy_(x), list(W.grids), ws)  # noqa: E731
    elif a.stage == "block":
        ws = vitq.workspace(vitq.block_workspace_bytes(n), dev)
        run = lambda: vitq.block_forward_(blk, x, cu, n, cs, ws)  # noqa: E731
    elif a.stage == "attention":
        qkv = wl.random_bf16((n, 3456), 1, 1.0).to(dev)
        vitq.rope2d_(qkv, cs, flags=vitq.V_FP16)
        out = torch.empty((n, 1152), dtype=torch.bfloat16, device=dev)
        run = lambda: vitq.attention_varlen(qkv, cu, n, out=out, flags=vitq.V_FP16)  # noqa: E731
    elif a.stage.startswith("gemm_"):
        name = a.stage[5:]
        w = t[name + "_w"]
        K = w.shape[1]
        act = wl.random_bf16((n, K), 2, 1.0).to(dev)
        qa, sa = vitq.quant_act(act)
        res = x if name in ("proj",) else (wl.random_bf16((n, 1152), 3).to(dev) if name == "fc2" else None)
        out = torch.empty((n, w.shape[0]), dtype=torch.bfloat16, device=dev)
        run = lambda: vitq.fp8_block_gemm(qa, sa, t[name + "_q"], t[name + "_s"], t[name + "_b"], res, out)  # noqa: E731
    elif a.stage.startswith("bf16_"):
        name = a.stage[5:]
        w = t[name + "_w"]
        act = wl.random_bf16((n, w.shape[1]), 2, 1.0).to(dev)
        out = torch.empty((n, w.shape[0]), dtype=torch.bfloat16, device=dev)
        run = lambda: vitq.bf16_gemm(act, w, t[name + "_b"], None, out)  # noqa: E731
    elif a.stage == "ln_quant":
        run = lambda: vitq.ln_quant(x, t["norm1_w"], t["norm1_b"])  # noqa: E731
    elif a.stage == "ln_quant_merger":
        xm = x.view(n // 4, 4608)
        g = (1 + wl.random_bf16((4608,), 6, 0.02).float()).to(torch.bfloat16).to(dev)
        b = wl.random_bf16((4608,), 7, 0.01).to(dev)
        run = lambda: vitq.ln_quant(xm, g, b)  # noqa: E731
    elif a.stage == "quant_act":
        run = lambda: vitq.quant_act(x)  # noqa: E731
    elif a.stage == "gelu_quant":
        f = wl.random_bf16((n, 4304), 4, 1.0).to(dev)
        run = lambda: vitq.gelu_quant(f)  # noqa: E731
    elif a.stage == "rope":
        qkv = wl.random_bf16((n, 3456), 5, 1.0).to(dev)
        run = lambda: vitq.rope2d_(qkv, cs)  # noqa: E731
    else:
        raise SystemExit(f"unknown stage {a.stage}")
    for _ in range(a.iters - 1):
        run()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("last_iter")
    run()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    assert vitq.device_error() == 0
    print(f"{a.stage}: {a.iters} iterations ok")


if __name__ == "__main__":
    main()
