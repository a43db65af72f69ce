"""Precision perturbations of the oracle, used to derive tolerances for composite outputs.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The FP8 block method re-quantises every activation to 3 mantissa bits, so a
difference of one bf16 ulp upstream flips an E4M3 code (a 1/16 relative jump)
with probability about 1/16; over a block these flips add up to a rel-L2 change
near 1e-2, and over the 27-block tower to several 1e-2 whatever the size of the
original difference.  A CUDA implementation cannot reproduce the oracle's
fp64 rounding of every intermediate, so block-, merger- and tower-level outputs
are compared against the drift the oracle itself shows when one of its
intermediate roundings is moved by a tiny amount.  (The pages show the same growth with
depth: FP8 against bf16 image-embedding cosines fall from block 8 to the last DeepStack
tap [FRT s4].)

Three perturbations are modelled, each a documented change of a rounding point:
  gemm_fp32_promotion : the per-128-K partial sums (exact) are scaled and summed
                        in fp32 instead of fp64 (a ~1e-7 relative change);
  attention_bf16_p    : softmax probabilities rounded to bf16 before the P.V
                        product, as a bf16 flash-attention kernel does;
  bf16_gemm_fp32      : the bf16 GEMMs accumulate in fp32 instead of fp64.
"""
from __future__ import annotations

import contextlib
import math

import numpy as np

from . import vit as ov
from .numerics import bf16_round, e4m3_decode


def fp8_block_gemm_fp32_promotion(qa, sa, qw, sw, bias=None, residual=None):
    """fp8_block_gemm with the K-block scaling and the outer sum in fp32 (the fp32
    accumulation of the FP8 GEMMs [FRT s1, s3])."""
    a = e4m3_decode(qa)
    w = e4m3_decode(qw)
    M, K = qa.shape
    N = qw.shape[0]
    acc = np.zeros((M, N), np.float32)
    wsc = np.repeat(sw, ov.QBLK, axis=0)[:N]
    for kb in range(-(-K // ov.QBLK)):
        ks = slice(kb * ov.QBLK, (kb + 1) * ov.QBLK)
        part = (a[:, ks] @ w[:, ks].T).astype(np.float32)
        acc = acc + part * (sa[kb][:, None].astype(np.float32) * wsc[:, kb][None, :].astype(np.float32))
    if bias is not None:
        acc = acc + np.asarray(bias, np.float32)[None, :]
    if residual is not None:
        acc = acc + np.asarray(residual, np.float32)
    return bf16_round(acc.astype(np.float64))


def attention_bf16_p(qkv, cu_seqlens, heads: int = 16, head_dim: int = 72, scale=None):
    """attention_varlen with P rounded to bf16 before the P.V product and the row sum (a bf16
    flash-attention kernel [FRT s3])."""
    qkv = np.asarray(qkv, np.float64)
    n = qkv.shape[0]
    scale = 1.0 / math.sqrt(head_dim) if scale is None else scale
    t = qkv.reshape(n, 3, heads, head_dim)
    out = np.zeros((n, heads, head_dim))
    cu = [int(c) for c in cu_seqlens]
    for a, b in zip(cu[:-1], cu[1:]):
        for h in range(heads):
            s = (t[a:b, 0, h] @ t[a:b, 1, h].T) * scale
            p = bf16_round(np.exp(s - s.max(axis=1, keepdims=True)))
            out[a:b, h] = (p @ t[a:b, 2, h]) / p.sum(axis=1, keepdims=True)
    return bf16_round(out.reshape(n, -1))


def bf16_gemm_fp32(a, w, bias=None, residual=None):
    """bf16_gemm with the product summed, and bias and residual added, in fp32 (the bf16
    linears of the first blocks and the mergers [FRT s4])."""
    acc = np.asarray(a, np.float32) @ np.asarray(w, np.float32).T
    if bias is not None:
        acc = acc + np.asarray(bias, np.float32)[None, :]
    if residual is not None:
        acc = acc + np.asarray(residual, np.float32)
    return bf16_round(acc.astype(np.float64))


@contextlib.contextmanager
def perturbed():
    """Within the context, the oracle's block/merger/tower use the perturbations
    (fp32 GEMM promotion or accumulation, bf16 attention probabilities), to measure
    the depth-growing drift the pages report for FP8 against bf16 [FRT s4]."""
    g, a, b = ov.fp8_block_gemm, ov.attention_varlen, ov.bf16_gemm
    ov.fp8_block_gemm, ov.attention_varlen, ov.bf16_gemm = fp8_block_gemm_fp32_promotion, attention_bf16_p, bf16_gemm_fp32
    try:
        yield
    finally:
        ov.fp8_block_gemm, ov.attention_varlen, ov.bf16_gemm = g, a, b
