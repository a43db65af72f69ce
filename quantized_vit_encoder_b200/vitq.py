"""ctypes binding of libvitq.so: the same entry points as include/vitq.h.

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels.  torch supplies device memory and the current CUDA
stream.  If the library is missing, loading raises; there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvitq.so")

HIDDEN, HEADS, HEAD_DIM, MLP, QKV = 1152, 16, 72, 4304, 3456
MERGE_IN, OUT_HIDDEN, N_BLOCKS = 4608, 2048, 27
PATCH_DIM, POS_GRID = 1536, 48
# vitq_status values (include/vitq.h)
OK, ERR_INVALID_ARG, ERR_SHAPE, ERR_ALIGN, ERR_ARCH, ERR_CUDA, ERR_WORKSPACE, ERR_DEVICE_TIMEOUT, ERR_RANGE = range(9)
STATUS = {OK: "ok", ERR_INVALID_ARG: "invalid argument", ERR_SHAPE: "unsupported shape",
          ERR_ALIGN: "pointer not 16-byte aligned", ERR_ARCH: "device is not sm_100", ERR_CUDA: "CUDA error",
          ERR_WORKSPACE: "workspace too small", ERR_DEVICE_TIMEOUT: "device pipeline wait timed out",
          ERR_RANGE: "value beyond the range of its format (clamped)"}

_vp, _i, _f, _sz = C.c_void_p, C.c_int, C.c_float, C.c_size_t


class BlockWeights(C.Structure):
    """vitq_block_weights: device pointers of one FP8 block."""
    _fields_ = [(n, _vp) for n in (
        "norm1_w", "norm1_b", "qkv_q", "qkv_s", "qkv_b", "proj_q", "proj_s", "proj_b",
        "norm2_w", "norm2_b", "fc1_q", "fc1_s", "fc1_b", "fc2_q", "fc2_s", "fc2_b")]


class MergerWeights(C.Structure):
    """vitq_merger_weights: device pointers of one FP8 merger."""
    _fields_ = [(n, _vp) for n in (
        "norm_w", "norm_b", "fc1_q", "fc1_s", "fc1_b", "fc2_q", "fc2_s", "fc2_b")]


class TowerWeights(C.Structure):
    """vitq_tower_weights: 27 blocks and 4 mergers."""
    _fields_ = [("blocks", BlockWeights * N_BLOCKS), ("mergers", MergerWeights * 4)]


BF16_HEAD_BLOCKS = 3


class BlockWeightsBf16(C.Structure):
    """vitq_block_weights_bf16: device pointers of one bf16 block."""
    _fields_ = [(n, _vp) for n in (
        "norm1_w", "norm1_b", "qkv_w", "qkv_b", "proj_w", "proj_b",
        "norm2_w", "norm2_b", "fc1_w", "fc1_b", "fc2_w", "fc2_b")]


class MergerWeightsBf16(C.Structure):
    """vitq_merger_weights_bf16: device pointers of one bf16 merger."""
    _fields_ = [(n, _vp) for n in ("norm_w", "norm_b", "fc1_w", "fc1_b", "fc2_w", "fc2_b")]


class TowerWeightsMixed(C.Structure):
    """vitq_tower_weights_mixed: bf16 blocks 1-3 and mergers, FP8 blocks 4-27."""
    _fields_ = [("head", BlockWeightsBf16 * BF16_HEAD_BLOCKS),
                ("blocks", BlockWeights * (N_BLOCKS - BF16_HEAD_BLOCKS)),
                ("mergers", MergerWeightsBf16 * 4)]


_SIGS = {
    "vit_quant_act": [_vp, _i, _i, _i, _vp, _vp, _i, _vp],
    "vit_quant_weight": [_vp, _i, _i, _vp, _vp, _vp],
    "vit_ln_quant": [_vp, _i, _i, _i, _vp, _vp, _f, _vp, _vp, _i, _vp],
    "vit_gelu_quant": [_vp, _i, _i, _i, _vp, _vp, _i, _vp],
    "fp8_block_gemm": [_vp, _vp, _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp],
    "bf16_gemm": [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp],
    "vit_rope_table": [_vp, _i, _f, _vp, _vp],
    "vit_rope2d": [_vp, _i, _vp, _i, _vp],
    "vit_positions": [_vp, _i, _vp, _vp, _vp],
    "vit_attention_varlen": [_vp, _i, _vp, _i, _i, _f, _i, _vp, _vp],
    "vit_block_forward": [C.POINTER(BlockWeights), _vp, _i, _vp, _i, _i, _vp, _vp, _sz, _vp],
    "vitq_block_workspace_bytes": [_i],
    "vit_merger_forward": [C.POINTER(MergerWeights), _vp, _i, _vp, _vp, _sz, _vp],
    "vit_merger_forward_static": [C.POINTER(MergerWeights), _vp, _i, _vp, _vp],
    "vitq_merger_workspace_bytes": [_i],
    "vit_tower_forward": [C.POINTER(TowerWeights), _vp, _vp, _i, C.POINTER(_vp), _vp, _sz, _vp],
    "vitq_tower_workspace_bytes": [_i, _i],
    "vit_block_forward_bf16": [C.POINTER(BlockWeightsBf16), _vp, _i, _vp, _i, _i, _vp, _vp, _sz, _vp],
    "vit_merger_forward_bf16": [C.POINTER(MergerWeightsBf16), _vp, _i, _vp, _vp, _sz, _vp],
    "vitq_merger_bf16_workspace_bytes": [_i],
    "vit_patch_embed": [_vp, _i, _vp, _i, _vp, _vp, _vp, _vp, _vp, _sz, _vp],
    "vitq_patch_embed_workspace_bytes": [_i],
    "vit_tower_forward_mixed": [C.POINTER(TowerWeightsMixed), _vp, _vp, _i, C.POINTER(_vp), _vp, _sz, _vp],
    "vitq_get_device_error": [_vp],
    "vitq_status_string": [_i],
    "vitq_launch_count": [],
    "vitq_profile_start": [],
    "vitq_profile_stop": [],
    "vitq_profile_get": [_i, C.POINTER(C.c_char_p), C.POINTER(C.c_float), C.POINTER(C.c_double),
                         C.POINTER(C.c_double)],
    "vitq_selftest_wait_timeout": [_i, _vp],
}
_RES = {"vitq_block_workspace_bytes": _sz, "vitq_merger_workspace_bytes": _sz,
        "vitq_merger_bf16_workspace_bytes": _sz, "vitq_patch_embed_workspace_bytes": _sz,
        "vitq_tower_workspace_bytes": _sz, "vitq_status_string": C.c_char_p,
        "vitq_launch_count": C.c_ulonglong, "vitq_profile_start": None}

_lib = None


def load(path: str = LIB_PATH):
    """Load libvitq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m quantized_vit_encoder_b200.build`")
        lib = C.CDLL(path)
        for name, args in _SIGS.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = _RES.get(name, _i)
        _lib = lib
    return _lib


class VitqError(RuntimeError):
    """A non-zero vitq_status, or a tensor argument the C side cannot take."""
    pass


def _check(status: int, what: str):
    if status != 0:
        raise VitqError(f"{what}: {STATUS.get(status, status)} ({status})")


def _p(t):
    return None if t is None else C.c_void_p(t.data_ptr())


_DEVICE_TYPE = "cuda"
_bf16, _f32, _u8, _i32 = torch.bfloat16, torch.float32, torch.uint8, torch.int32


def _arg(t, name, dtype, shape=None, rows=False):
    """Check a tensor before its pointer crosses the ABI: device memory, the dtype
    the C side reads, the shape (None entries are free) and a dense layout
    (rows=True: each row dense, the row stride is passed to the C side)."""
    if not isinstance(t, torch.Tensor):
        raise VitqError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.device.type != _DEVICE_TYPE:
        raise VitqError(f"{name}: tensor on {t.device}; the library reads device memory only")
    if t.dtype != dtype:
        raise VitqError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if shape is not None and (t.dim() != len(shape) or
                              any(w is not None and w != d for w, d in zip(shape, t.shape))):
        raise VitqError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    dense = (t.dim() == 2 and t.stride(1) == 1 and t.stride(0) >= t.shape[1]) if rows else t.is_contiguous()
    if not dense:
        raise VitqError(f"{name}: strides {t.stride()} are not a dense{' row' if rows else ''} layout")
    return t


def _cs(cos_sin, n):
    _arg(cos_sin, "cos_sin", _f32, (None, 72))
    if cos_sin.shape[0] < n:
        raise VitqError(f"cos_sin: {cos_sin.shape[0]} rows for {n} tokens")
    return cos_sin


def _cu(cu_seqlens):
    _arg(cu_seqlens, "cu_seqlens", _i32, (None,))
    if cu_seqlens.shape[0] < 1:
        raise VitqError("cu_seqlens: needs at least one entry")
    return cu_seqlens


def _ws(ws):
    return _arg(ws, "ws", _u8, (None,))


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def launch_count() -> int:
    """Kernel launches issued by the library since it was loaded."""
    return int(load().vitq_launch_count())


def device_error(stream=None) -> int:
    """Synchronise the stream, then read and clear the device error word: OK, ERR_DEVICE_TIMEOUT
    after a bounded wait timed out, ERR_RANGE after a clamped fp16 v value, ERR_CUDA if
    synchronising failed."""
    return int(load().vitq_get_device_error(_stream(stream)))


def profile_start():
    """Start bracketing every library launch with CUDA events (not during stream capture)."""
    load().vitq_profile_start()


def profile_stop() -> list:
    """Per-launch records since profile_start: [(kernel name, ms, flops, bytes), ...]."""
    lib = load()
    n = lib.vitq_profile_stop()
    if n < 0:
        _check(-n, "vitq_profile_stop")
    out = []
    name, ms, fl, by = C.c_char_p(), C.c_float(), C.c_double(), C.c_double()
    for i in range(n):
        _check(lib.vitq_profile_get(i, C.byref(name), C.byref(ms), C.byref(fl), C.byref(by)), "vitq_profile_get")
        out.append((name.value.decode(), float(ms.value), float(fl.value), float(by.value)))
    return out


def selftest_wait_timeout(limit_us: int = 20000, stream=None):
    """Launch a kernel whose pipeline wait can never complete; it gives up after limit_us."""
    _check(load().vitq_selftest_wait_timeout(limit_us, _stream(stream)), "vitq_selftest_wait_timeout")


# ---------------------------------------------------------------- stages

def _scales(nkb, M, device):
    lds = (M + 3) // 4 * 4
    return torch.zeros((nkb, lds), dtype=torch.float32, device=device), lds


def quant_act(x: torch.Tensor, stream=None):
    """1x128 FP8 quantisation of bf16 x [M, K] -> (codes uint8 [M, K], scales fp32 [ceil(K/128), M_pad4])."""
    M, K = _arg(x, "x", _bf16, (None, None), rows=True).shape
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    s, lds = _scales((K + 127) // 128, M, x.device)
    _check(load().vit_quant_act(_p(x), M, K, x.stride(0), _p(q), _p(s), lds, _stream(stream)), "vit_quant_act")
    return q, s


def quant_weight(w: torch.Tensor, stream=None):
    """128x128-block FP8 quantisation of bf16 w [N, K] -> (codes [N, K], scales [ceil(N/128), ceil(K/128)])."""
    N, K = _arg(w, "w", _bf16, (None, None)).shape
    q = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    s = torch.zeros(((N + 127) // 128, (K + 127) // 128), dtype=torch.float32, device=w.device)
    _check(load().vit_quant_weight(_p(w), N, K, _p(q), _p(s), _stream(stream)), "vit_quant_weight")
    return q, s


def ln_quant(x, gamma, beta, eps: float = 1e-6, stream=None):
    """LayerNorm of bf16 x [M, K] (rows dense), rounded to bf16 and 1x128 FP8-quantised -> (codes, scales)."""
    M, K = _arg(x, "x", _bf16, (None, None), rows=True).shape
    _arg(gamma, "gamma", _bf16, (K,))
    _arg(beta, "beta", _bf16, (K,))
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    s, lds = _scales((K + 127) // 128, M, x.device)
    _check(load().vit_ln_quant(_p(x), M, K, x.stride(0), _p(gamma), _p(beta), eps, _p(q), _p(s), lds,
                               _stream(stream)), "vit_ln_quant")
    return q, s


def gelu_quant(f, stream=None):
    """GELU(tanh) of bf16 f [M, K] (rows dense), rounded to bf16 and 1x128 FP8-quantised -> (codes, scales)."""
    M, K = _arg(f, "f", _bf16, (None, None), rows=True).shape
    q = torch.empty((M, K), dtype=torch.uint8, device=f.device)
    s, lds = _scales((K + 127) // 128, M, f.device)
    _check(load().vit_gelu_quant(_p(f), M, K, f.stride(0), _p(q), _p(s), lds, _stream(stream)), "vit_gelu_quant")
    return q, s


def fp8_block_gemm(qa, sa, qw, sw, bias=None, residual=None, out=None, stream=None):
    """bf16 C [M, N] = block-scaled FP8 product (+ bias) (+ residual)."""
    M, K = _arg(qa, "qa", _u8, (None, None)).shape
    N = _arg(qw, "qw", _u8, (None, K)).shape[0]
    _arg(sa, "sa", _f32, ((K + 127) // 128, None), rows=True)
    if sa.shape[1] < M:
        raise VitqError(f"sa: {sa.shape[1]} columns for {M} rows")
    _arg(sw, "sw", _f32, ((N + 127) // 128, (K + 127) // 128))
    if bias is not None:
        _arg(bias, "bias", _bf16, (N,))
    if residual is not None:
        _arg(residual, "residual", _bf16, (M, N))
    if out is not None:
        _arg(out, "out", _bf16, (M, N))
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=qa.device)
    _check(load().fp8_block_gemm(_p(qa), _p(sa), sa.stride(0), _p(qw), _p(sw), _p(bias), _p(residual), _p(out),
                                 M, N, K, _stream(stream)), "fp8_block_gemm")
    return out


def bf16_gemm(a, w, bias=None, residual=None, out=None, stream=None):
    """bf16 C [M, N] = a [M, K] w[N, K]^T (+ bias) (+ residual), fp32 accumulation."""
    M, K = _arg(a, "a", _bf16, (None, None)).shape
    N = _arg(w, "w", _bf16, (None, K)).shape[0]
    if bias is not None:
        _arg(bias, "bias", _bf16, (N,))
    if residual is not None:
        _arg(residual, "residual", _bf16, (M, N))
    if out is not None:
        _arg(out, "out", _bf16, (M, N))
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    _check(load().bf16_gemm(_p(a), _p(w), _p(bias), _p(residual), _p(out), M, N, K, _stream(stream)), "bf16_gemm")
    return out


def rope_table(pos_hw: torch.Tensor, theta: float = 10000.0, stream=None):
    """cos / sin table fp32 [n, 72] for int32 (row, col) positions [n, 2]."""
    n = _arg(pos_hw, "pos_hw", _i32, (None, 2)).shape[0]
    cs = torch.empty((n, 72), dtype=torch.float32, device=pos_hw.device)
    _check(load().vit_rope_table(_p(pos_hw), n, theta, _p(cs), _stream(stream)), "vit_rope_table")
    return cs


V_FP16 = 1


def rope2d_(qkv: torch.Tensor, cos_sin: torch.Tensor, flags: int = 0, stream=None):
    """In-place 2D rotary on the q, k parts of qkv; flags=V_FP16 also converts v to fp16 in place."""
    _cs(cos_sin, _arg(qkv, "qkv", _bf16, (None, QKV)).shape[0])
    _check(load().vit_rope2d(_p(qkv), qkv.shape[0], _p(cos_sin), flags, _stream(stream)), "vit_rope2d")
    return qkv


def positions(grids, device="cuda", stream=None):
    """(pos_hw int32 [n, 2], cu_seqlens int32 [n_images + 1]) for packed grids [(h, w), ...]."""
    g = (C.c_int32 * (2 * len(grids)))(*[v for hw in grids for v in hw])
    n = sum(h * w for h, w in grids)
    pos = torch.empty((n, 2), dtype=torch.int32, device=device)
    cu = torch.empty((len(grids) + 1,), dtype=torch.int32, device=device)
    _check(load().vit_positions(C.cast(g, C.c_void_p), len(grids), _p(pos), _p(cu), _stream(stream)),
           "vit_positions")
    return pos, cu


def attention_varlen(qkv, cu_seqlens, max_seqlen: int, scale: float | None = None, out=None, flags: int = 0,
                     stream=None):
    """Block-diagonal attention over bf16 qkv [n, 3456] with int32 cu_seqlens -> bf16 [n, 1152]."""
    n = _arg(qkv, "qkv", _bf16, (None, QKV)).shape[0]
    _cu(cu_seqlens)
    if out is None:
        out = torch.empty((n, HIDDEN), dtype=torch.bfloat16, device=qkv.device)
    _arg(out, "out", _bf16, (n, HIDDEN))
    if scale is None:
        scale = 1.0 / math.sqrt(HEAD_DIM)
    _check(load().vit_attention_varlen(_p(qkv), n, _p(cu_seqlens), cu_seqlens.shape[0] - 1, max_seqlen, scale,
                                       flags, _p(out), _stream(stream)), "vit_attention_varlen")
    return out


# ---------------------------------------------------------------- layers

BLOCK_SHAPES = {"norm1_w": (HIDDEN,), "norm1_b": (HIDDEN,), "qkv_w": (QKV, HIDDEN), "qkv_b": (QKV,),
                "proj_w": (HIDDEN, HIDDEN), "proj_b": (HIDDEN,), "norm2_w": (HIDDEN,), "norm2_b": (HIDDEN,),
                "fc1_w": (MLP, HIDDEN), "fc1_b": (MLP,), "fc2_w": (HIDDEN, MLP), "fc2_b": (HIDDEN,)}
MERGER_SHAPES = {"norm_w": (MERGE_IN,), "norm_b": (MERGE_IN,), "fc1_w": (MERGE_IN, MERGE_IN),
                 "fc1_b": (MERGE_IN,), "fc2_w": (OUT_HIDDEN, MERGE_IN), "fc2_b": (OUT_HIDDEN,)}


def _weights(params: dict, shapes: dict, device) -> dict:
    """The bf16 weights a block or merger needs, on the device, dense, shape-checked."""
    missing = [k for k in shapes if k not in params]
    if missing:
        raise VitqError(f"weights missing: {missing}")
    t = {k: params[k].to(device).contiguous() for k in shapes}
    for k, shp in shapes.items():
        _arg(t[k], k, _bf16, shp)
    return t


def _x(x, name="x"):
    return _arg(x, name, _bf16, (None, HIDDEN)).shape[0]


def _merged_out(out, n, name="out"):
    if n % 4:
        raise VitqError(f"{n} tokens: the 2x2 merger takes a multiple of 4")
    return _arg(out, name, _bf16, (n // 4, OUT_HIDDEN))


def _taps(taps, n):
    if len(taps) != 4:
        raise VitqError(f"taps: {len(taps)} tensors, the tower has 4 mergers")
    for i, t in enumerate(taps):
        _merged_out(t, n, f"taps[{i}]")

class DeviceBlock:
    """Device-resident block weights (bf16 vectors, FP8 codes, fp32 scales) and their C struct."""

    def __init__(self, params: dict, device="cuda", stream=None):
        t = _weights(params, BLOCK_SHAPES, device)
        self.t = t
        for name in ("qkv", "proj", "fc1", "fc2"):
            t[name + "_q"], t[name + "_s"] = quant_weight(t[name + "_w"], stream)
        self.struct = BlockWeights(**{f: t[f].data_ptr() for f, _ in BlockWeights._fields_})


class DeviceMerger:
    """Device-resident merger weights (bf16 vectors, FP8 codes, fp32 scales) and their C struct."""

    def __init__(self, params: dict, device="cuda", stream=None):
        t = _weights(params, MERGER_SHAPES, device)
        self.t = t
        for name in ("fc1", "fc2"):
            t[name + "_q"], t[name + "_s"] = quant_weight(t[name + "_w"], stream)
        self.struct = MergerWeights(**{f: t[f].data_ptr() for f, _ in MergerWeights._fields_})


class DeviceBlockBf16:
    """Device-resident bf16 block weights (no quantisation) and their C struct."""

    def __init__(self, params: dict, device="cuda"):
        self.t = _weights(params, BLOCK_SHAPES, device)
        self.struct = BlockWeightsBf16(**{f: self.t[f].data_ptr() for f, _ in BlockWeightsBf16._fields_})


class DeviceMergerBf16:
    """Device-resident bf16 merger weights and their C struct."""

    def __init__(self, params: dict, device="cuda"):
        self.t = _weights(params, MERGER_SHAPES, device)
        self.struct = MergerWeightsBf16(**{f: self.t[f].data_ptr() for f, _ in MergerWeightsBf16._fields_})


class DeviceTowerMixed:
    """Blocks 1-3 and the mergers bf16 (DeviceBlockBf16 / DeviceMergerBf16), blocks 4-27 FP8 (DeviceBlock)."""

    def __init__(self, head, blocks, mergers):
        self.head, self.blocks, self.mergers = head, blocks, mergers
        self.struct = TowerWeightsMixed()
        for i, b in enumerate(head):
            self.struct.head[i] = b.struct
        for i, b in enumerate(blocks):
            self.struct.blocks[i] = b.struct
        for i, m in enumerate(mergers):
            self.struct.mergers[i] = m.struct


def block_forward_bf16_(blk: DeviceBlockBf16, x, cu_seqlens, max_seqlen, cos_sin, ws, stream=None):
    """In-place bf16 block forward on bf16 x [n, 1152]."""
    _cs(cos_sin, _x(x))
    _cu(cu_seqlens)
    _ws(ws)
    _check(load().vit_block_forward_bf16(C.byref(blk.struct), _p(x), x.shape[0], _p(cu_seqlens),
                                         cu_seqlens.shape[0] - 1, max_seqlen, _p(cos_sin), _p(ws), ws.numel(),
                                         _stream(stream)), "vit_block_forward_bf16")
    return x


def merger_bf16_workspace_bytes(n: int) -> int:
    """Workspace bytes of vit_merger_forward_bf16 at n input tokens (0 if n is out of range)."""
    return int(load().vitq_merger_bf16_workspace_bytes(n))


def merger_forward_bf16(mg: DeviceMergerBf16, x, ws, out=None, stream=None):
    """bf16 2x2 merger of bf16 x [n, 1152] -> [n/4, 2048]."""
    n = _x(x)
    _ws(ws)
    if out is None:
        out = torch.empty((n // 4, OUT_HIDDEN), dtype=torch.bfloat16, device=x.device)
    _merged_out(out, n)
    _check(load().vit_merger_forward_bf16(C.byref(mg.struct), _p(x), n, _p(out), _p(ws), ws.numel(),
                                          _stream(stream)), "vit_merger_forward_bf16")
    return out


def tower_forward_mixed_(tower: DeviceTowerMixed, x, grids, ws, taps=None, stream=None):
    """In-place mixed-precision tower forward; returns the four taps [n/4, 2048]."""
    n = _x(x)
    _ws(ws)
    if taps is None:
        taps = [torch.empty((n // 4, OUT_HIDDEN), dtype=torch.bfloat16, device=x.device) for _ in range(4)]
    _taps(taps, n)
    g = (C.c_int32 * (2 * len(grids)))(*[v for hw in grids for v in hw])
    tp = (C.c_void_p * 4)(*[t.data_ptr() for t in taps])
    _check(load().vit_tower_forward_mixed(C.byref(tower.struct), _p(x), C.cast(g, C.c_void_p), len(grids), tp,
                                          _p(ws), ws.numel(), _stream(stream)), "vit_tower_forward_mixed")
    return taps


def patch_embed(pixels, grids, w, b, pos_table, out=None, ws=None, stream=None):
    """bf16 x [n, 1152] = pixels [n, 1536] . w^T + b + interpolated position embedding."""
    n = _arg(pixels, "pixels", _bf16, (None, PATCH_DIM)).shape[0]
    _arg(w, "w", _bf16, (HIDDEN, PATCH_DIM))
    _arg(b, "b", _bf16, (HIDDEN,))
    _arg(pos_table, "pos_table", _bf16, (POS_GRID * POS_GRID, HIDDEN))
    if out is None:
        out = torch.empty((n, HIDDEN), dtype=torch.bfloat16, device=pixels.device)
    _arg(out, "out", _bf16, (n, HIDDEN))
    if ws is None:
        ws = workspace(int(load().vitq_patch_embed_workspace_bytes(n)), pixels.device)
    _ws(ws)
    g = (C.c_int32 * (2 * len(grids)))(*[v for hw in grids for v in hw])
    _check(load().vit_patch_embed(_p(pixels), n, C.cast(g, C.c_void_p), len(grids), _p(w), _p(b), _p(pos_table),
                                  _p(out), _p(ws), ws.numel(), _stream(stream)), "vit_patch_embed")
    return out


def block_workspace_bytes(n: int) -> int:
    """Workspace bytes of vit_block_forward at n tokens (0 if n is out of range)."""
    return int(load().vitq_block_workspace_bytes(n))


def merger_workspace_bytes(n: int) -> int:
    """Workspace bytes of vit_merger_forward at n input tokens (0 if n is out of range)."""
    return int(load().vitq_merger_workspace_bytes(n))


def tower_workspace_bytes(n: int, n_images: int) -> int:
    """Workspace bytes of the tower at up to n tokens in up to n_images images (0 if out of range)."""
    return int(load().vitq_tower_workspace_bytes(n, n_images))


def workspace(nbytes: int, device="cuda"):
    """A uint8 device buffer of nbytes (at least 1) to pass as a workspace."""
    return torch.empty((max(nbytes, 1),), dtype=torch.uint8, device=device)


def block_forward_(blk: DeviceBlock, x, cu_seqlens, max_seqlen, cos_sin, ws, stream=None):
    """In-place block forward on bf16 x [n, 1152]."""
    _cs(cos_sin, _x(x))
    _cu(cu_seqlens)
    _ws(ws)
    _check(load().vit_block_forward(C.byref(blk.struct), _p(x), x.shape[0], _p(cu_seqlens), cu_seqlens.shape[0] - 1,
                                    max_seqlen, _p(cos_sin), _p(ws), ws.numel(), _stream(stream)),
           "vit_block_forward")
    return x


def merger_forward(mg: DeviceMerger, x, ws, out=None, stream=None):
    """FP8 2x2 merger of bf16 x [n, 1152] -> [n/4, 2048]."""
    n = _x(x)
    _ws(ws)
    if out is None:
        out = torch.empty((n // 4, OUT_HIDDEN), dtype=torch.bfloat16, device=x.device)
    _merged_out(out, n)
    _check(load().vit_merger_forward(C.byref(mg.struct), _p(x), n, _p(out), _p(ws), ws.numel(), _stream(stream)),
           "vit_merger_forward")
    return out


MERGER_STATIC_MAX_TOKENS = 4096


def merger_forward_static(mg: DeviceMerger, x, out):
    """vit_merger_forward_static: the merger with the library's fixed scratch
    (no workspace, no allocation); out must be given, bf16 [n/4, 2048]."""
    _merged_out(out, _x(x))
    _check(load().vit_merger_forward_static(C.byref(mg.struct), _p(x), x.shape[0], _p(out), _stream(None)),
           "vit_merger_forward_static")
    return out


class DeviceTower:
    """27 DeviceBlock and 4 DeviceMerger objects and the vitq_tower_weights struct over them."""

    def __init__(self, blocks, mergers):
        self.blocks, self.mergers = blocks, mergers
        self.struct = TowerWeights()
        for i, b in enumerate(blocks):
            self.struct.blocks[i] = b.struct
        for i, m in enumerate(mergers):
            self.struct.mergers[i] = m.struct


def tower_forward_(tower: DeviceTower, x, grids, ws, taps=None, stream=None):
    """In-place tower forward on bf16 x [n, 1152]; returns the four tap tensors [n/4, 2048]."""
    n = _x(x)
    _ws(ws)
    if taps is None:
        taps = [torch.empty((n // 4, OUT_HIDDEN), dtype=torch.bfloat16, device=x.device) for _ in range(4)]
    _taps(taps, n)
    g = (C.c_int32 * (2 * len(grids)))(*[v for hw in grids for v in hw])
    tp = (C.c_void_p * 4)(*[t.data_ptr() for t in taps])
    _check(load().vit_tower_forward(C.byref(tower.struct), _p(x), C.cast(g, C.c_void_p), len(grids), tp, _p(ws),
                                    ws.numel(), _stream(stream)), "vit_tower_forward")
    return taps
