"""include/vitq.h from plain C: the header compiles as strict C99, a C program links
libvitq.so and gets the host-side answers (status strings, workspace sizes, argument
and size-limit errors), and the weight structs have the same layout in C as in the
Python binding's ctypes declarations.  Host only: nothing here reaches a device."""
import ctypes
import os
import shutil
import subprocess

import pytest

from quantized_vit_encoder_b200 import vitq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SRC = r"""
#include <stdio.h>
#include <stddef.h>
#include "vitq.h"

#define OFF(T, f) printf(#T "." #f " %zu\n", offsetof(T, f))

int main(void) {
  printf("sizeof.block %zu\n", sizeof(vitq_block_weights));
  printf("sizeof.merger %zu\n", sizeof(vitq_merger_weights));
  printf("sizeof.tower %zu\n", sizeof(vitq_tower_weights));
  printf("sizeof.block_bf16 %zu\n", sizeof(vitq_block_weights_bf16));
  printf("sizeof.merger_bf16 %zu\n", sizeof(vitq_merger_weights_bf16));
  printf("sizeof.tower_mixed %zu\n", sizeof(vitq_tower_weights_mixed));
  OFF(vitq_block_weights, fc2_b);
  OFF(vitq_merger_weights, fc2_s);
  OFF(vitq_tower_weights, mergers);
  OFF(vitq_tower_weights_mixed, blocks);
  OFF(vitq_tower_weights_mixed, mergers);
  printf("ws.block %zu\n", vitq_block_workspace_bytes(6256));
  printf("ws.merger %zu\n", vitq_merger_workspace_bytes(6256));
  printf("ws.tower %zu\n", vitq_tower_workspace_bytes(9164, 4));
  printf("ws.over %zu\n", vitq_block_workspace_bytes(VITQ_MAX_ROWS + 1));
  printf("err.null %d\n", vit_quant_act(NULL, 4, 128, 128, NULL, NULL, 4, NULL));
  printf("err.rows %d\n", vit_rope2d((void*)4096, VITQ_MAX_ROWS + 1, (const float*)4096, 0, NULL));
  printf("str.6 %s\n", vitq_status_string(VITQ_ERR_WORKSPACE));
  return 0;
}
"""


@pytest.fixture(scope="module")
def c_output(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    from quantized_vit_encoder_b200 import build
    lib = build.build(verbose=False)
    d = tmp_path_factory.mktemp("c_consumer")
    src = d / "consumer.c"
    src.write_text(C_SRC)
    exe = d / "consumer"
    libdir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), "-L", libdir, "-l:" + os.path.basename(lib), "-Wl,-rpath," + libdir]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    return dict(line.split(" ", 1) for line in r.stdout.splitlines())


def test_structs_match_the_ctypes_binding(c_output):
    o = c_output
    assert int(o["sizeof.block"]) == ctypes.sizeof(vitq.BlockWeights)
    assert int(o["sizeof.merger"]) == ctypes.sizeof(vitq.MergerWeights)
    assert int(o["sizeof.tower"]) == ctypes.sizeof(vitq.TowerWeights)
    assert int(o["sizeof.block_bf16"]) == ctypes.sizeof(vitq.BlockWeightsBf16)
    assert int(o["sizeof.merger_bf16"]) == ctypes.sizeof(vitq.MergerWeightsBf16)
    assert int(o["sizeof.tower_mixed"]) == ctypes.sizeof(vitq.TowerWeightsMixed)
    assert int(o["vitq_block_weights.fc2_b"]) == vitq.BlockWeights.fc2_b.offset
    assert int(o["vitq_merger_weights.fc2_s"]) == vitq.MergerWeights.fc2_s.offset
    assert int(o["vitq_tower_weights.mergers"]) == vitq.TowerWeights.mergers.offset
    assert int(o["vitq_tower_weights_mixed.blocks"]) == vitq.TowerWeightsMixed.blocks.offset
    assert int(o["vitq_tower_weights_mixed.mergers"]) == vitq.TowerWeightsMixed.mergers.offset


def test_host_answers_from_c(c_output):
    o = c_output
    assert int(o["ws.block"]) == vitq.block_workspace_bytes(6256)
    assert int(o["ws.merger"]) == vitq.merger_workspace_bytes(6256)
    assert int(o["ws.tower"]) == vitq.tower_workspace_bytes(9164, 4)
    assert int(o["ws.over"]) == 0
    assert int(o["err.null"]) == 1 and int(o["err.rows"]) == 2
    assert o["str.6"] == "workspace too small"
