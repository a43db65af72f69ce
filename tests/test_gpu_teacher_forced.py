"""Teacher-forced parity of the whole tower, block by block and stage by stage.

The 27-block tower is chaotic under FP8 re-quantisation: a one-ulp bf16
difference anywhere flips E4M3 codes downstream, so the end-to-end taps of any
implementation that is not bit-identical to the oracle drift apart with depth
(tests/test_gpu_layers.py bounds that drift).  These tests pin the tower
instead by teacher forcing: the GPU runs the tower block by block and stage by
stage through the C ABI, and every stage of every checked block and merger is
compared with the oracle's stage fed the GPU's own input to that stage:

  * FP8 codes and scales (LayerNorm+quant, attention-output quant, GELU+quant):
    bit-exact;
  * bf16 stage outputs (the four GEMMs, rotary, attention): rel-L2 <= 1e-2 and
    |gpu - oracle| <= max(3e-2, one bf16 ulp of the oracle value) per element.

The stage chain is first checked to reproduce, bit for bit, the output of
vit_block_forward (so the stages are the block), and the block chain to
reproduce the taps of vit_tower_forward (so the blocks are the tower).  The
three workloads are the 16x16 image (all 27 blocks and all 4 mergers), the
46x136 image (blocks 1, 14 and 27 and the final merger) and the packed
four-image batch with per-image input scales 0.1 / 1 / 10 / 1 (blocks 1 and 27
and the final merger).  "Qwen3-VL-8B on RTX 5090", section 3 (block chain,
DeepStack taps, 2x2 merger) and section 5 (one attention window per image).
"""
import numpy as np
import pytest
import torch

from oracle import vit as ov
from quantized_vit_encoder_b200 import workloads as wl

pytestmark = pytest.mark.gpu

REL_L2 = 1e-2
MAX_ABS = 3e-2


def f64(t):
    return t.detach().float().cpu().double().numpy()


def bf16_ulp(v):
    """Spacing of bf16 numbers at |v| (2^(e - 7) for |v| in [2^e, 2^(e+1)))."""
    a = np.maximum(np.abs(np.asarray(v, np.float64)), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


def check_bf16_stage(got, ref, what):
    """The per-stage bound: rel-L2 <= 1e-2 and max-abs <= max(3e-2, 1 ulp) per element."""
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    worst = float((np.abs(got - ref) / np.maximum(MAX_ABS, bf16_ulp(ref))).max())
    assert rel <= REL_L2 and worst <= 1.0, f"{what}: rel_l2 {rel:.3e}, max-abs / allowed {worst:.2f}"
    return rel


def check_codes(q_gpu, s_gpu, q_ref, s_ref, what):
    """FP8 codes and scales bit-exact (GPU scales are [ceil(K/128), M_pad4])."""
    m = q_ref.shape[0]
    qg = q_gpu.cpu().numpy()
    sg = s_gpu.cpu().numpy()[:, :m]
    n_bad = int((qg != q_ref).sum())
    assert n_bad == 0, f"{what}: {n_bad} of {q_ref.size} codes differ"
    assert np.array_equal(sg.view(np.uint32), np.asarray(s_ref, np.float32).view(np.uint32)), f"{what}: scales"


def oracle_block_weights(seed):
    return ov.quantize_block_weights({k: f64(v) for k, v in wl.block_params(seed).items()})


def oracle_merger_weights(seed):
    return ov.quantize_merger_weights({k: f64(v) for k, v in wl.merger_params(seed).items()})


def gpu_block_stages(blk, x, cu, max_len, cs):
    """One FP8 block through the stage entry points, in the order and with the arguments
    vit_block_forward uses; returns every stage's output (x is not modified)."""
    from quantized_vit_encoder_b200 import vitq
    t = blk.t
    st = {"x": x}
    st["q1"], st["s1"] = vitq.ln_quant(x, t["norm1_w"], t["norm1_b"])
    st["qkv"] = vitq.fp8_block_gemm(st["q1"], st["s1"], t["qkv_q"], t["qkv_s"], t["qkv_b"])
    st["qkv_rot"] = vitq.rope2d_(st["qkv"].clone(), cs, flags=vitq.V_FP16)
    st["attn"] = vitq.attention_varlen(st["qkv_rot"], cu, max_len, flags=vitq.V_FP16)
    st["qo"], st["so"] = vitq.quant_act(st["attn"])
    st["x1"] = vitq.fp8_block_gemm(st["qo"], st["so"], t["proj_q"], t["proj_s"], t["proj_b"], residual=x)
    st["q2"], st["s2"] = vitq.ln_quant(st["x1"], t["norm2_w"], t["norm2_b"])
    st["f"] = vitq.fp8_block_gemm(st["q2"], st["s2"], t["fc1_q"], t["fc1_s"], t["fc1_b"])
    st["qg"], st["sg"] = vitq.gelu_quant(st["f"])
    st["x2"] = vitq.fp8_block_gemm(st["qg"], st["sg"], t["fc2_q"], t["fc2_s"], t["fc2_b"], residual=st["x1"])
    return st


def rotated_qkv_values(qkv_rot):
    """The values the attention reads: q, k bf16 and v stored as fp16 (exact from bf16)."""
    v = f64(qkv_rot)
    v[:, 2304:] = qkv_rot[:, 2304:].contiguous().view(torch.float16).float().cpu().double().numpy()
    return v


def check_block_teacher_forced(st, ow, cu_ref, pos_ref, what):
    """Each stage of one GPU block against the oracle's stage fed the GPU's input to it."""
    x = f64(st["x"])
    q1, s1 = ov.ln_quant(x, ow["norm1_w"], ow["norm1_b"])
    check_codes(st["q1"], st["s1"], q1, s1, f"{what} LN1+quant")
    qkv = ov.fp8_block_gemm(q1, s1, ow["qkv_q"], ow["qkv_s"], bias=ow["qkv_b"])
    check_bf16_stage(f64(st["qkv"]), qkv, f"{what} QKV GEMM")
    qkv_in = f64(st["qkv"])
    rot = ov.apply_rope_qkv(qkv_in, pos_ref)
    got_rot = rotated_qkv_values(st["qkv_rot"])
    check_bf16_stage(got_rot[:, :2304], rot[:, :2304], f"{what} rotary q, k")
    # v is the round-to-nearest fp16 value of the bf16 v (exact for |v| >= 2^-14)
    v_f16 = st["qkv"][:, 2304:].float().half().double().cpu().numpy()
    assert np.array_equal(got_rot[:, 2304:], v_f16), f"{what}: v is not the fp16 rounding of the bf16 v"
    attn = ov.attention_varlen(got_rot, cu_ref)
    check_bf16_stage(f64(st["attn"]), attn, f"{what} attention")
    qo, so = ov.quant_act(f64(st["attn"]))
    check_codes(st["qo"], st["so"], qo, so, f"{what} O quant")
    x1 = ov.fp8_block_gemm(qo, so, ow["proj_q"], ow["proj_s"], bias=ow["proj_b"], residual=x)
    check_bf16_stage(f64(st["x1"]), x1, f"{what} proj GEMM + residual")
    q2, s2 = ov.ln_quant(f64(st["x1"]), ow["norm2_w"], ow["norm2_b"])
    check_codes(st["q2"], st["s2"], q2, s2, f"{what} LN2+quant")
    f = ov.fp8_block_gemm(q2, s2, ow["fc1_q"], ow["fc1_s"], bias=ow["fc1_b"])
    check_bf16_stage(f64(st["f"]), f, f"{what} fc1 GEMM")
    qg, sg = ov.gelu_quant(f64(st["f"]))
    check_codes(st["qg"], st["sg"], qg, sg, f"{what} GELU+quant")
    x2 = ov.fp8_block_gemm(qg, sg, ow["fc2_q"], ow["fc2_s"], bias=ow["fc2_b"], residual=f64(st["x1"]))
    check_bf16_stage(f64(st["x2"]), x2, f"{what} fc2 GEMM + residual")


def gpu_merger_stages(mg, x):
    from quantized_vit_encoder_b200 import vitq
    t = mg.t
    xm = x.view(x.shape[0] // 4, 4 * wl.HIDDEN)
    st = {"x": x}
    st["q1"], st["s1"] = vitq.ln_quant(xm, t["norm_w"], t["norm_b"])
    st["h"] = vitq.fp8_block_gemm(st["q1"], st["s1"], t["fc1_q"], t["fc1_s"], t["fc1_b"])
    st["qg"], st["sg"] = vitq.gelu_quant(st["h"])
    st["out"] = vitq.fp8_block_gemm(st["qg"], st["sg"], t["fc2_q"], t["fc2_s"], t["fc2_b"])
    return st


def check_merger_teacher_forced(st, ow, what):
    xm = f64(st["x"]).reshape(-1, 4 * wl.HIDDEN)
    q1, s1 = ov.ln_quant(xm, ow["norm_w"], ow["norm_b"])
    check_codes(st["q1"], st["s1"], q1, s1, f"{what} LN(4608)+quant")
    h = ov.fp8_block_gemm(q1, s1, ow["fc1_q"], ow["fc1_s"], bias=ow["fc1_b"])
    check_bf16_stage(f64(st["h"]), h, f"{what} fc1 GEMM")
    qg, sg = ov.gelu_quant(f64(st["h"]))
    check_codes(st["qg"], st["sg"], qg, sg, f"{what} GELU+quant")
    out = ov.fp8_block_gemm(qg, sg, ow["fc2_q"], ow["fc2_s"], bias=ow["fc2_b"])
    check_bf16_stage(f64(st["out"]), out, f"{what} fc2 GEMM")


def run_tower_teacher_forced(W, check_blocks, check_mergers):
    """Runs the tower block by block (vit_block_forward / vit_merger_forward) and checks:
    the chain's taps equal vit_tower_forward's bit for bit; the stage chain of each block
    in check_blocks equals vit_block_forward's output bit for bit and matches the oracle
    stage by stage; likewise the mergers in check_mergers (0-based tap index)."""
    from quantized_vit_encoder_b200 import vitq
    grids = list(W.grids)
    n = W.n_tokens
    max_len = max(h * w for h, w in grids)
    blocks = [vitq.DeviceBlock(wl.block_params(wl.block_seed(W, b))) for b in range(wl.N_BLOCKS)]
    mergers = [vitq.DeviceMerger(wl.merger_params(wl.merger_seed(W, t))) for t in range(4)]
    x0 = wl.make_input(W).cuda()
    ws = vitq.workspace(vitq.tower_workspace_bytes(n, len(grids)))
    taps_tower = vitq.tower_forward_(vitq.DeviceTower(blocks, mergers), x0.clone(), grids, ws)
    assert vitq.device_error() == 0

    pos, cu = vitq.positions(grids)
    cs = vitq.rope_table(pos)
    pos_ref, cu_ref = ov.packed_positions(grids)
    assert np.array_equal(pos.cpu().numpy(), pos_ref) and np.array_equal(cu.cpu().numpy(), np.asarray(cu_ref))
    wsb = vitq.workspace(vitq.block_workspace_bytes(n))
    wsm = vitq.workspace(vitq.merger_workspace_bytes(n))
    x = x0.clone()
    tap = 0
    for b in range(1, wl.N_BLOCKS + 1):
        blk = blocks[b - 1]
        if b in check_blocks:
            st = gpu_block_stages(blk, x.clone(), cu, max_len, cs)
        vitq.block_forward_(blk, x, cu, max_len, cs, wsb)
        if b in check_blocks:
            assert torch.equal(st["x2"], x), f"block {b}: stage chain differs from vit_block_forward"
            ow = oracle_block_weights(wl.block_seed(W, b - 1))
            for name in ("qkv", "proj", "fc1", "fc2"):
                assert np.array_equal(blk.t[name + "_q"].cpu().numpy(), ow[name + "_q"]), f"block {b} {name} codes"
            check_block_teacher_forced(st, ow, cu_ref, pos_ref, f"{W.name} block {b}")
            del st
        if tap < 4 and b == wl.TAP_AFTER[tap]:
            out = vitq.merger_forward(mergers[tap], x, wsm)
            assert torch.equal(out, taps_tower[tap]), f"tap {tap}: block chain differs from vit_tower_forward"
            if tap in check_mergers:
                st = gpu_merger_stages(mergers[tap], x)
                assert torch.equal(st["out"], out), f"merger {tap}: stage chain differs from vit_merger_forward"
                check_merger_teacher_forced(st, oracle_merger_weights(wl.merger_seed(W, tap)),
                                            f"{W.name} merger {tap}")
            tap += 1
    assert tap == 4
    assert vitq.device_error() == 0


def test_tower_16x16_every_block_and_merger(lib):
    """All 27 blocks and all 4 mergers of a 16x16 tower, every stage teacher-forced."""
    W = wl.Workload("tower_16x16", ((16, 16),), wl.N_BLOCKS, True, seed_base=5400)
    run_tower_teacher_forced(W, set(range(1, wl.N_BLOCKS + 1)), {0, 1, 2, 3})


def test_tower_46x136_blocks_1_14_27(lib):
    """The full-size 46x136 tower (6256 patches): blocks 1, 14 and 27 and the final merger."""
    run_tower_teacher_forced(wl.WORKLOADS["tower_46x136"], {1, 14, 27}, {3})


def test_tower_packed4_mixed_scales(lib):
    """The packed batch 54x18 + 46x136 + 24x38 + 32x32 (9164 patches) with per-image input
    scales 0.1 / 1 / 10 / 1: blocks 1 and 27 and the final merger."""
    run_tower_teacher_forced(wl.WORKLOADS["tower_packed4"], {1, 27}, {3})
