"""Host-side checks of the C ABI (no GPU needed): the library builds, loads and
exports every entry point that include/vitq.h declares."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vitq.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?(?:int|size_t|unsigned long long|char\s*\*|const char\s*\*)\s*\**\s*(\w+)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def built_lib():
    from quantized_vit_encoder_b200 import build
    path = build.build(verbose=False)
    return ctypes.CDLL(path)


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("vit_quant_act", "fp8_block_gemm", "vit_rope2d", "vit_attention_varlen",
                     "vit_block_forward", "vit_merger_forward", "vit_tower_forward", "vit_quant_weight",
                     "vit_rope_table", "vitq_tower_workspace_bytes", "vitq_get_device_error",
                     "vitq_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(built_lib):
    missing = [n for n in _declared() if not hasattr(built_lib, n)]
    assert not missing, missing


def test_host_only_calls(built_lib):
    lib = built_lib
    lib.vitq_status_string.restype = ctypes.c_char_p
    assert lib.vitq_status_string(0) == b"ok"
    assert lib.vitq_status_string(6) == b"workspace too small"
    lib.vitq_block_workspace_bytes.restype = ctypes.c_size_t
    lib.vitq_tower_workspace_bytes.restype = ctypes.c_size_t
    b = lib.vitq_block_workspace_bytes(6256)
    # codes (4304/row) + scales + qkv + attn + x1 + fc1 out, all bf16 or bytes
    assert b >= 6256 * (4304 + 2 * (3456 + 1152 + 1152 + 4304))
    assert lib.vitq_tower_workspace_bytes(9164, 4) > lib.vitq_block_workspace_bytes(9164)


def test_invalid_arguments_rejected_before_any_launch(built_lib):
    """Null pointers and bad shapes return a status on the host; nothing reaches CUDA."""
    lib = built_lib
    v = ctypes.c_void_p
    assert lib.vit_quant_act(None, 4, 128, 128, None, None, 4, None) == 1
    fake = v(4096)
    assert lib.fp8_block_gemm(fake, fake, 8, fake, fake, None, None, fake, 8, 64, 100, None) == 2   # K % 16
    assert lib.fp8_block_gemm(v(4100), fake, 8, fake, fake, None, None, fake, 8, 64, 128, None) == 3  # align
    assert lib.vit_merger_forward(None, fake, 8, fake, fake, 1 << 30, None) == 1
    g = (ctypes.c_int32 * 2)(3, 4)
    assert lib.vit_positions(ctypes.cast(g, v), 0, fake, fake, None) == 1


def test_oversized_grids_rejected_on_the_host(built_lib):
    """Grid sizes whose patch count leaves the int range are a shape error, found before any launch."""
    lib = built_lib
    v = ctypes.c_void_p
    fake = v(4096)
    for hw in ((65536, 65536), (1 << 16, 1 << 15), (40000, 30000)):
        g = (ctypes.c_int32 * 2)(*hw)
        assert lib.vit_positions(ctypes.cast(g, v), 1, fake, fake, None) == 2
    g = (ctypes.c_int32 * 4)(20000, 30000, 20000, 30000)      # each fits, the total does not
    assert lib.vit_positions(ctypes.cast(g, v), 2, fake, fake, None) == 2
