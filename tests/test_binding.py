"""The Python binding's argument checks and marshalling, on CPU.

The binding hands raw pointers to the C library, so a host tensor, a wrong dtype or
a strided view would reach a kernel as a bad pointer or a misread layout.  These
tests run every binding call the GPU tests and the benchmark make, with CPU tensors
of the same shapes, against a stub of the library that records the arguments (the
device type the binding accepts is switched to "cpu" for them), and check that each
call passes its checks and marshals the sizes and strides the C side expects.  The
negative cases run with the real device rule and check that nothing reaches the
library.
"""
import ctypes

import pytest
import torch

from quantized_vit_encoder_b200 import vitq
from quantized_vit_encoder_b200 import workloads as wl


class _Stub:
    """Records each library call; workspace sizes come from the real library (host-only)."""

    def __init__(self, real):
        self.calls, self.real = [], real

    def __getattr__(self, name):
        if name.endswith("_workspace_bytes"):
            return getattr(self.real, name)

        def fn(*args):
            self.calls.append((name, args))
            return 0
        return fn


def _v(a):
    return a.value if isinstance(a, (ctypes.c_void_p, ctypes.c_int, ctypes.c_float)) else a


@pytest.fixture
def stub(monkeypatch):
    real = vitq.load()
    s = _Stub(real)
    monkeypatch.setattr(vitq, "_lib", s)
    monkeypatch.setattr(vitq, "_stream", lambda stream=None: None)
    return s


@pytest.fixture
def on_cpu(monkeypatch, stub):
    monkeypatch.setattr(vitq, "_DEVICE_TYPE", "cpu")
    return stub


def _bf(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def _last(stub, name):
    calls = [a for n, a in stub.calls if n == name]
    assert calls, f"{name} was not called"
    return [_v(a) for a in calls[-1]]


def test_stage_calls_marshal_sizes_and_strides(on_cpu):
    x = _bf(200, 1152)
    vitq.quant_act(x)
    a = _last(on_cpu, "vit_quant_act")
    assert a[1:4] == [200, 1152, 1152] and a[6] == 200
    wide = _bf(10, 4608)[:, :1152]                       # rows dense, row stride 4608
    vitq.quant_act(wide)
    assert _last(on_cpu, "vit_quant_act")[1:4] == [10, 1152, 4608]
    vitq.quant_weight(_bf(384, 640))
    assert _last(on_cpu, "vit_quant_weight")[1:3] == [384, 640]
    vitq.ln_quant(x, _bf(1152), _bf(1152))
    assert _last(on_cpu, "vit_ln_quant")[1:4] == [200, 1152, 1152]
    vitq.gelu_quant(_bf(7, 4304))
    assert _last(on_cpu, "vit_gelu_quant")[1:4] == [7, 4304, 4304]

    M, N, K = 200, 384, 640
    qa, qw = torch.zeros((M, K), dtype=torch.uint8), torch.zeros((N, K), dtype=torch.uint8)
    sa, sw = torch.zeros((5, 200)), torch.zeros((3, 5))
    vitq.fp8_block_gemm(qa, sa, qw, sw)
    a = _last(on_cpu, "fp8_block_gemm")
    assert a[2] == 200 and a[8:11] == [M, N, K] and a[5] is None and a[6] is None
    sa_pad = torch.zeros((5, 204))
    vitq.fp8_block_gemm(qa, sa_pad, qw, sw, _bf(N), _bf(M, N))
    a = _last(on_cpu, "fp8_block_gemm")
    assert a[2] == 204 and a[5] is not None and a[6] is not None
    vitq.bf16_gemm(_bf(M, K), _bf(N, K), _bf(N), _bf(M, N))
    assert _last(on_cpu, "bf16_gemm")[5:8] == [M, N, K]

    pos = torch.zeros((300, 2), dtype=torch.int32)
    cs = vitq.rope_table(pos)
    assert cs.shape == (300, 72) and _last(on_cpu, "vit_rope_table")[1] == 300
    qkv = _bf(300, 3456)
    vitq.rope2d_(qkv, cs, flags=vitq.V_FP16)
    assert _last(on_cpu, "vit_rope2d")[1] == 300 and _last(on_cpu, "vit_rope2d")[3] == vitq.V_FP16
    cu = torch.tensor([0, 100, 300], dtype=torch.int32)
    out = vitq.attention_varlen(qkv, cu, 200)
    a = _last(on_cpu, "vit_attention_varlen")
    assert out.shape == (300, 1152) and a[1] == 300 and a[3] == 2 and a[4] == 200


def test_layer_calls_pass_their_checks(on_cpu):
    blk = vitq.DeviceBlock(wl.block_params(1), device="cpu")
    mg = vitq.DeviceMerger(wl.merger_params(2), device="cpu")
    n = 256
    x, cs, cu = _bf(n, 1152), torch.zeros((n, 72)), torch.tensor([0, n], dtype=torch.int32)
    ws = vitq.workspace(vitq.block_workspace_bytes(n), "cpu")
    vitq.block_forward_(blk, x, cu, n, cs, ws)
    a = _last(on_cpu, "vit_block_forward")
    assert a[2] == n and a[4] == 1 and a[5] == n and a[8] == ws.numel()
    out = vitq.merger_forward(mg, x, vitq.workspace(vitq.merger_workspace_bytes(n), "cpu"))
    assert out.shape == (n // 4, 2048) and _last(on_cpu, "vit_merger_forward")[2] == n
    vitq.merger_forward_static(mg, x, _bf(n // 4, 2048))
    assert _last(on_cpu, "vit_merger_forward_static")[2] == n

    tower = vitq.DeviceTower([blk] * wl.N_BLOCKS, [mg] * 4)
    tws = vitq.workspace(vitq.tower_workspace_bytes(n, 1), "cpu")
    taps = vitq.tower_forward_(tower, x, [(16, 16)], tws)
    assert len(taps) == 4 and all(t.shape == (n // 4, 2048) for t in taps)
    a = _last(on_cpu, "vit_tower_forward")
    assert a[3] == 1 and a[6] == tws.numel()

    b16 = vitq.DeviceBlockBf16(wl.block_params(3), "cpu")
    m16 = vitq.DeviceMergerBf16(wl.merger_params(4), "cpu")
    vitq.block_forward_bf16_(b16, x, cu, n, cs, ws)
    vitq.merger_forward_bf16(m16, x, vitq.workspace(vitq.merger_bf16_workspace_bytes(n), "cpu"))
    # the mixed tower reuses the FP8 blocks' bf16 tensors, as the benchmark does
    head = [vitq.DeviceBlockBf16({k: blk.t[k] for k in vitq.BLOCK_SHAPES}, "cpu")] * vitq.BF16_HEAD_BLOCKS
    mixed = vitq.DeviceTowerMixed(head, [blk] * (wl.N_BLOCKS - vitq.BF16_HEAD_BLOCKS), [m16] * 4)
    vitq.tower_forward_mixed_(mixed, x, [(16, 16)], tws)
    assert _last(on_cpu, "vit_tower_forward_mixed")[3] == 1

    p = wl.patch_params(5)
    pix = _bf(n, 1536)
    emb = vitq.patch_embed(pix, [(16, 16)], p["w"], p["b"], p["pos"], ws=torch.zeros(n * 2304, dtype=torch.uint8))
    assert emb.shape == (n, 1152) and _last(on_cpu, "vit_patch_embed")[1] == n


def _rejects(stub, fn, *args, **kw):
    before = len(stub.calls)
    with pytest.raises(vitq.VitqError):
        fn(*args, **kw)
    assert len(stub.calls) == before, "a rejected call reached the library"


def test_host_tensors_never_reach_the_library(stub):
    _rejects(stub, vitq.quant_act, _bf(4, 128))
    _rejects(stub, vitq.bf16_gemm, _bf(8, 64), _bf(64, 64))
    _rejects(stub, vitq.rope_table, torch.zeros((4, 2), dtype=torch.int32))
    _rejects(stub, vitq.DeviceBlockBf16, wl.block_params(1), "cpu")


def test_wrong_dtype_shape_or_layout_rejected(on_cpu):
    s = on_cpu
    _rejects(s, vitq.quant_act, torch.zeros((4, 128)))                       # fp32, not bf16
    _rejects(s, vitq.quant_act, _bf(128, 4).t())                             # column-major
    _rejects(s, vitq.quant_weight, _bf(256, 128)[::2])                       # row-strided, no ld argument
    _rejects(s, vitq.ln_quant, _bf(4, 128), _bf(64), _bf(128))               # gamma length
    qa, qw = torch.zeros((8, 128), dtype=torch.uint8), torch.zeros((64, 128), dtype=torch.uint8)
    _rejects(s, vitq.fp8_block_gemm, qa, torch.zeros((1, 4)), qw, torch.zeros((1, 1)))   # sa has 4 < 8 columns
    _rejects(s, vitq.fp8_block_gemm, qa, torch.zeros((1, 8)), qw, torch.zeros((1, 2)))   # sw shape
    _rejects(s, vitq.fp8_block_gemm, qa, torch.zeros((1, 8), dtype=torch.float64), qw, torch.zeros((1, 1)))
    _rejects(s, vitq.bf16_gemm, _bf(8, 64), _bf(64, 32))                     # K mismatch
    _rejects(s, vitq.rope2d_, _bf(10, 3456), torch.zeros((9, 72)))           # table too short
    _rejects(s, vitq.attention_varlen, _bf(10, 3456), torch.tensor([0, 10]), 10)   # int64 cu_seqlens
    _rejects(s, vitq.attention_varlen, _bf(10, 1152), torch.tensor([0, 10], dtype=torch.int32), 10)
    p = wl.block_params(1)
    bad = dict(p, fc1_w=_bf(4304, 1152).t().contiguous())                   # transposed weight
    _rejects(s, vitq.DeviceBlock, bad, "cpu")
    _rejects(s, vitq.DeviceBlock, {k: v for k, v in p.items() if k != "qkv_b"}, "cpu")
    mg = vitq.DeviceMerger(wl.merger_params(2), device="cpu")
    _rejects(s, vitq.merger_forward, mg, _bf(6, 1152), torch.zeros(64, dtype=torch.uint8))     # 6 % 4
    _rejects(s, vitq.merger_forward_static, mg, _bf(8, 1152), _bf(3, 2048))
    _rejects(s, vitq.merger_forward, mg, _bf(8, 1152), torch.zeros(16))     # fp32 workspace
    tower = vitq.DeviceTower([vitq.DeviceBlock(p, device="cpu")] * wl.N_BLOCKS, [mg] * 4)
    _rejects(s, vitq.tower_forward_, tower, _bf(16, 1152), [(4, 4)], torch.zeros(64, dtype=torch.uint8),
             [_bf(4, 2048)] * 3)
