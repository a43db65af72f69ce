"""Device clock traces of CTA 0 of the FP8 GEMM and the attention kernel (development tool).

Builds libvitq_trace.so (the library compiled with -DVITQ_TRACE: each kernel's CTA 0
stores clock64() at its pipeline events into a device table), runs one traced launch
after three warm-up launches, reads the table back with vitq_trace_read and prints the
median cycles between events. Needs a B200; the timings of a trace build are slower than
the normal build's, the event intervals are what it is for.

    python -m quantized_vit_encoder_b200.trace_case gemm        # fc1 and fc2 at 6256 rows
    python -m quantized_vit_encoder_b200.trace_case attention   # one 46x136 image, fp16 v
"""
from __future__ import annotations

import argparse
import ctypes as C
import os
import subprocess

import numpy as np
import torch

from . import build, vitq
from . import workloads as wl

TRACE_LIB = os.path.join(build.PKG, "libvitq_trace.so")
TAGS, PER_TAG = 32, 4096


def load_trace_lib():
    """Build the trace library if its sources are newer, and load it as the binding's library."""
    deps = [os.path.join(build.CSRC, s) for s in build.SOURCES] + [os.path.join(build.ROOT, "include", "vitq.h")]
    if not os.path.exists(TRACE_LIB) or any(os.path.getmtime(d) > os.path.getmtime(TRACE_LIB) for d in deps):
        subprocess.run(build.nvcc_cmd(out=TRACE_LIB, extra=["-DVITQ_TRACE"]), check=True)
    if vitq._lib is not None:
        raise RuntimeError("the binding already loaded another library in this process")
    return vitq.load(TRACE_LIB)


def read_table(lib) -> np.ndarray:
    buf = (C.c_ulonglong * (TAGS * PER_TAG))()
    n = lib.vitq_trace_read(buf, TAGS * PER_TAG)
    if n != TAGS * PER_TAG:
        raise RuntimeError(f"vitq_trace_read returned {n}")
    return np.frombuffer(buf, dtype=np.uint64).reshape(TAGS, PER_TAG).astype(np.int64)


def _med(v) -> int:
    return int(np.median(v)) if len(v) else -1


def gemm(lib):
    """Per-K-block events of the FP8 GEMM (tags: 1 producer issues loads, 2 MMA thread has a
    free TMEM buffer, 3 operands landed, 4 epilogue waits for a partial, 5 partial ready,
    6 partial consumed, 7 K loop of a tile done, 9 staging tile free)."""
    n = 6256
    W = wl.WORKLOADS["block_46x136"]
    blk = vitq.DeviceBlock(wl.block_params(wl.block_seed(W, 0)), "cuda")
    t = blk.t
    for name in ("fc1", "fc2"):
        w = t[name + "_w"]
        N, K = w.shape
        act = wl.random_bf16((n, K), 2, 1.0).cuda()
        qa, sa = vitq.quant_act(act)
        res = wl.random_bf16((n, wl.HIDDEN), 3).cuda() if name == "fc2" else None
        out = torch.empty((n, N), dtype=torch.bfloat16, device="cuda")
        run = lambda: vitq.fp8_block_gemm(qa, sa, t[name + "_q"], t[name + "_s"], t[name + "_b"], res, out)  # noqa: E731
        for _ in range(3):
            run()
        torch.cuda.synchronize()
        read_table(lib)                                   # clears the table
        run()
        torch.cuda.synchronize()
        tr = read_table(lib)
        nkb = (K + 127) // 128
        cnt = int((tr[3] > 0).sum())
        R = range(nkb, min(cnt - 1, 4 * nkb))            # K blocks of tiles 2-4 of CTA 0

        def d(a, b):
            return [int(tr[b, c] - tr[a, c]) for c in R if tr[a, c] and tr[b, c]]
        print(f"== {name}: N={N} K={K} nkb={nkb} K blocks traced={cnt}")
        print("  K-block period (3 -> next 3):", _med([int(tr[3, c + 1] - tr[3, c]) for c in R if tr[3, c + 1]]))
        print("  MMA thread, previous block's issue + buffer wait (prev 3 -> 2):",
              _med([int(tr[2, c] - tr[3, c - 1]) for c in R]), " operand wait (2 -> 3):", _med(d(2, 3)))
        print("  epilogue wait for the partial (4 -> 5):", _med(d(4, 5)), " promotion (5 -> 6):", _med(d(5, 6)),
              " operands landed -> partial ready (3 -> 5):", _med(d(3, 5)))
        print("  tile period (7):", [int(tr[7, i] - tr[7, i - 1]) for i in range(1, 4) if tr[7, i]])
        assert vitq.device_error() == 0


def attention(lib):
    """Per-step events of the two Q tiles x = A, B of attention CTA 0 (tags + x: 10 S issued,
    12 P.V issued, 14 P complete (MMA side), 16 S buffer free, 20 S ready, 22 max known,
    24 P written, 26 S in registers, 28 turn for the exponentials)."""
    n = 6256
    qkv = wl.random_bf16((n, 3456), 1, 1.0).cuda()
    pos, cu = vitq.positions([(46, 136)], "cuda")
    cs = vitq.rope_table(pos)
    vitq.rope2d_(qkv, cs, flags=vitq.V_FP16)
    out = torch.empty((n, wl.HIDDEN), dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        vitq.attention_varlen(qkv, cu, n, out=out, flags=vitq.V_FP16)
    torch.cuda.synchronize()
    read_table(lib)
    vitq.attention_varlen(qkv, cu, n, out=out, flags=vitq.V_FP16)
    torch.cuda.synchronize()
    t = read_table(lib)
    steps = int((t[20] > 0).sum())            # 128-key steps recorded for tile A
    R = range(2, max(3, steps - 2))
    print(f"{steps} steps; tile A step period (S ready to S ready, 128 keys):",
          _med([t[20, j + 1] - t[20, j] for j in R]))
    print("exponential phase (turn -> P written): A", _med([t[24, j] - t[28, j] for j in R]),
          "B", _med([t[25, j] - t[29, j] for j in R]))
    print("S ready -> S in registers", _med([t[26, j] - t[20, j] for j in R]),
          " -> max known", _med([t[22, j] - t[26, j] for j in R]),
          " -> turn", _med([t[28, j] - t[22, j] for j in R]))
    print("P written -> seen by the MMA thread", _med([t[14, j] - t[24, j] for j in R]),
          " S buffer free -> next S issued", _med([t[10, j + 1] - t[16, j] for j in R]),
          " S issued -> S ready", _med([t[20, j + 1] - t[10, j + 1] for j in R]))
    assert vitq.device_error() == 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=("gemm", "attention"))
    a = ap.parse_args()
    if not torch.cuda.is_available():
        raise SystemExit("trace_case needs a CUDA device")
    lib = load_trace_lib()
    lib.vitq_trace_read.argtypes = [C.POINTER(C.c_ulonglong), C.c_int]
    lib.vitq_trace_read.restype = C.c_int
    {"gemm": gemm, "attention": attention}[a.case](lib)


if __name__ == "__main__":
    main()
