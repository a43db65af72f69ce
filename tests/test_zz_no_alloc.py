"""vit_merger_forward_static (the merger with the library's own fixed scratch,
no workspace and no allocation) against vit_merger_forward on the same inputs.

Both entry points launch the same kernels with the same shapes, so the outputs
must agree within the merger's test tolerance (in practice bit for bit).  Two
calls of different sizes run back to back, so scratch left over from the first
call cannot leak into the second.  This file is collected last so that it also
runs after every other test has used the library."""
import ctypes

import pytest

from quantized_vit_encoder_b200 import workloads as wl

MAX_TOKENS = 4096
# Merger outputs are bf16 [n/4, 2048]; identical kernels on identical inputs.
ATOL = 0.0


def _fake_weights():
    from quantized_vit_encoder_b200 import vitq
    w = vitq.MergerWeights()
    for name, _ in vitq.MergerWeights._fields_:
        setattr(w, name, 4096)
    return w


def test_static_merger_rejects_sizes_beyond_its_scratch():
    """Host-side checks only: too many tokens is refused before any device work."""
    from quantized_vit_encoder_b200 import build, vitq
    lib = ctypes.CDLL(build.build(verbose=False))
    fn = lib.vit_merger_forward_static
    fn.argtypes = [ctypes.POINTER(vitq.MergerWeights), ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                   ctypes.c_void_p]
    w = _fake_weights()
    fake = ctypes.c_void_p(4096)
    assert fn(ctypes.byref(w), fake, MAX_TOKENS + 4, fake, None) == vitq.ERR_WORKSPACE
    assert fn(ctypes.byref(w), fake, 1 << 30, fake, None) == vitq.ERR_WORKSPACE
    assert fn(ctypes.byref(w), fake, 6, fake, None) == vitq.ERR_SHAPE       # n % 4 != 0
    assert fn(None, fake, 8, fake, None) == vitq.ERR_INVALID_ARG
    assert fn(ctypes.byref(w), None, 8, fake, None) == vitq.ERR_INVALID_ARG


@pytest.mark.gpu
def test_static_merger_matches_workspace_merger(lib):
    import torch
    from quantized_vit_encoder_b200 import vitq
    assert vitq.MERGER_STATIC_MAX_TOKENS == MAX_TOKENS
    mg = vitq.DeviceMerger(wl.merger_params(5151))
    for n_tokens, seed in ((MAX_TOKENS, 11), (972, 12)):
        x = wl.random_bf16((n_tokens, 1152), seed, 2.0).cuda()
        ws = vitq.workspace(vitq.merger_workspace_bytes(n_tokens))
        want = vitq.merger_forward(mg, x, ws)
        out = torch.full((n_tokens // 4, 2048), float("nan"), dtype=torch.bfloat16, device="cuda")
        got = vitq.merger_forward_static(mg, x, out)
        torch.cuda.synchronize()
        assert vitq.device_error() == 0
        assert torch.isfinite(got.float()).all()
        diff = (got.float() - want.float()).abs().max().item()
        assert diff <= ATOL, (n_tokens, diff)
    with pytest.raises(vitq.VitqError):
        big = torch.zeros((MAX_TOKENS + 4, 1152), dtype=torch.bfloat16, device="cuda")
        vitq.merger_forward_static(mg, big, torch.empty((MAX_TOKENS // 4 + 1, 2048), dtype=torch.bfloat16,
                                                        device="cuda"))
