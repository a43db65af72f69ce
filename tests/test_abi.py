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
    names = re.findall(r"^\s*(?:const\s+)?(?:int|size_t|void|unsigned long long|char\s*\*|const char\s*\*)\s*\**\s*(\w+)\s*\(",
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
    assert lib.vitq_status_string(8).startswith(b"value beyond the range")
    assert lib.vitq_status_string(9) == b"unknown status"
    lib.vitq_block_workspace_bytes.restype = ctypes.c_size_t
    lib.vitq_tower_workspace_bytes.restype = ctypes.c_size_t
    b = lib.vitq_block_workspace_bytes(6256)
    # codes (4304/row) + scales + qkv + attn + x1 + fc1 out, all bf16 or bytes
    assert b >= 6256 * (4304 + 2 * (3456 + 1152 + 1152 + 4304))
    assert lib.vitq_tower_workspace_bytes(9164, 4) > lib.vitq_block_workspace_bytes(9164)
    # an empty profile needs no device: 0 records, and record 0 does not exist
    lib.vitq_profile_start()
    assert lib.vitq_profile_stop() == 0
    name, ms, fl, by = ctypes.c_char_p(), ctypes.c_float(), ctypes.c_double(), ctypes.c_double()
    ref = ctypes.byref
    assert lib.vitq_profile_get(0, ref(name), ref(ms), ref(fl), ref(by)) == 1


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
    g = (ctypes.c_int32 * 4)(4096, 3000, 4096, 3000)      # each fits, the total does not
    assert lib.vit_positions(ctypes.cast(g, v), 2, fake, fake, None) == 2


MAX_ROWS, MAX_DIM = 1 << 24, 1 << 16


def test_header_size_limits_match():
    src = open(HEADER).read()
    assert re.search(r"#define VITQ_MAX_ROWS \(1 << 24\)", src)
    assert re.search(r"#define VITQ_MAX_DIM \(1 << 16\)", src)


def test_size_limits_rejected_on_the_host(built_lib):
    """Counts past VITQ_MAX_ROWS / VITQ_MAX_DIM are a shape error at every entry point,
    found before any device query (so the status comes back here, without a GPU), and
    the workspace sizes are 0 past the limit but not at it."""
    lib = built_lib
    v, i = ctypes.c_void_p, ctypes.c_int
    fake = v(4096)
    R, D = MAX_ROWS + 1, MAX_DIM + 8
    assert lib.vit_quant_act(fake, R, 128, 128, fake, fake, R, None) == 2
    assert lib.vit_ln_quant(fake, R, 128, 128, fake, fake, ctypes.c_float(1e-6), fake, fake, R, None) == 2
    assert lib.vit_gelu_quant(fake, R, 128, 128, fake, fake, R, None) == 2
    assert lib.vit_gelu_quant(fake, 8, MAX_DIM + 16, MAX_DIM + 16, fake, fake, 8, None) == 2
    assert lib.vit_quant_weight(fake, D, 128, fake, fake, None) == 2
    assert lib.vit_quant_weight(fake, 128, MAX_DIM + 16, fake, fake, None) == 2
    # M near the int maximum: (M + 127) / 128 must never be formed
    for m, n, k in ((R, 64, 128), ((1 << 31) - 1, 64, 128), (8, D, 128), (8, 64, MAX_DIM + 16)):
        assert lib.fp8_block_gemm(fake, fake, m, fake, fake, None, None, fake, m, n, k, None) == 2
        assert lib.bf16_gemm(fake, fake, None, None, fake, m, n, k, None) == 2
    assert lib.vit_rope_table(fake, R, ctypes.c_float(10000.0), fake, None) == 2
    assert lib.vit_rope2d(fake, R, fake, 0, None) == 2
    assert lib.vit_attention_varlen(fake, R, fake, 1, 16, ctypes.c_float(0.1), 0, fake, None) == 2
    assert lib.vit_attention_varlen(fake, 16, fake, 1, R, ctypes.c_float(0.1), 0, fake, None) == 2

    from quantized_vit_encoder_b200 import vitq
    bw = vitq.BlockWeights(*([4096] * len(vitq.BlockWeights._fields_)))
    mw = vitq.MergerWeights(*([4096] * len(vitq.MergerWeights._fields_)))
    bw16 = vitq.BlockWeightsBf16(*([4096] * len(vitq.BlockWeightsBf16._fields_)))
    mw16 = vitq.MergerWeightsBf16(*([4096] * len(vitq.MergerWeightsBf16._fields_)))
    big = ctypes.c_size_t(1 << 62)
    ref = ctypes.byref
    assert lib.vit_block_forward(ref(bw), fake, R, fake, 1, 16, fake, fake, big, None) == 2
    assert lib.vit_block_forward(ref(bw), fake, 16, fake, 1, R, fake, fake, big, None) == 2
    assert lib.vit_block_forward_bf16(ref(bw16), fake, R, fake, 1, 16, fake, fake, big, None) == 2
    assert lib.vit_merger_forward(ref(mw), fake, MAX_ROWS + 4, fake, fake, big, None) == 2
    assert lib.vit_merger_forward_bf16(ref(mw16), fake, MAX_ROWS + 4, fake, fake, big, None) == 2
    g = (ctypes.c_int32 * 2)(4096, 4098)                      # 16785408 patches, one image
    assert lib.vit_patch_embed(fake, 4096 * 4098, ctypes.cast(g, v), 1, fake, fake, fake, fake, fake, big,
                               None) == 2

    for name in ("vitq_block_workspace_bytes", "vitq_merger_workspace_bytes",
                 "vitq_patch_embed_workspace_bytes", "vitq_merger_bf16_workspace_bytes"):
        f = getattr(lib, name)
        f.restype, f.argtypes = ctypes.c_size_t, [i]
        assert f(MAX_ROWS) > 0 and f(MAX_ROWS + 4) == 0 and f(-4) == 0, name
    f = lib.vitq_tower_workspace_bytes
    f.restype, f.argtypes = ctypes.c_size_t, [i, i]
    assert f(MAX_ROWS, 4) > 0 and f(MAX_ROWS + 4, 4) == 0


_DECL = re.compile(r"^(?:const\s+)?(?:int|size_t|void|char\s*\*|const char\s*\*|unsigned long long)\s*\**\s*(\w+)\s*\(")


def _doc_blocks():
    """(name, the comment block that documents it) for every function the header declares:
    the comment directly above the declaration, or above a run of declarations (and
    #defines) that it heads, in which case the block must name the function."""
    lines = open(HEADER).read().splitlines()
    out = []
    for i, ln in enumerate(lines):
        m = _DECL.match(ln)
        if not m:
            continue
        j, grouped = i - 1, False
        while j >= 0 and not lines[j].rstrip().endswith("*/"):
            assert lines[j].startswith(("#define", " ")) or _DECL.match(lines[j]), \
                f"{m.group(1)}: no comment directly above ({lines[j]!r})"
            grouped = grouped or bool(_DECL.match(lines[j]))
            j -= 1
        k = j
        while k >= 0 and "/*" not in lines[k]:
            k -= 1
        doc = "\n".join(lines[k:j + 1])
        assert not grouped or m.group(1) in doc, f"{m.group(1)}: shares a comment that does not name it"
        out.append((m.group(1), doc))
    return out


def test_every_declared_function_is_documented():
    blocks = _doc_blocks()
    assert {n for n, _ in blocks} == set(_declared())
    for name, doc in blocks:
        assert len(doc) > 40, name
        if name.startswith("vit_") or name in ("fp8_block_gemm", "bf16_gemm"):
            # the operation's source section, or a pointer to the entry point that gives it
            assert re.search(r"\[(FRT|VE|TRT)\]|\bas vit_|merger above|no counterpart", doc), name
