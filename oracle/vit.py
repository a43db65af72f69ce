"""Stage-by-stage CPU definition of the FP8 ViT block, 2x2 merger and tower.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources (web pages; the section named is where the step is described):
  [FRT]  "Qwen3-VL-8B on RTX 5090 (NVFP4 language stack + FP8 ViT)":
         section 1 "Headline performance" (FP8 block-128 ViT GEMMs, quant fused
         into LayerNorm/GELU, bias adds fused), section 3 "Inference
         architecture" (block order, 2D rotate_half RoPE, FA2 full
         bidirectional attention, GELU(tanh), DeepStack taps, 2x2 merger,
         per-token / per-128-K-block FP8 activation quant), section 5 "Notes &
         limitations" (one attention window per image, cu_seqlens).
  [VE]   "spark_model/layers/vision_encoder.rs": the ViTBlock / MergerLayer /
         VisionEncoder structs (dims 1152/16/72/4304/2048, deepstack indexes
         [8, 16, 24] plus the final merger after block 27, rope_inv_freq of
         head_dim/4 entries).
  [TRT]  "qwen3_omni: record why FP8 is not shipped", section "Recipe that was
         measured": FP8 scale = amax / 448.

Readings where the pages are silent (each is listed with its reason in the
design notes):
  * activation quant: s = fl32(amax / 448) per row per 128 columns, code =
    E4M3_RNE_sat(fl32(y / s)) with IEEE fp32 division; a zero scale gives zero
    codes.  Weights: the same per 128x128 block.
  * GEMM: exact per-128-K partial sums (fp64 is exact for sums of 128
    E4M3*E4M3 products), scaled by sA*sW and summed over K blocks in fp64;
    bias and residual are added before the single bf16 rounding.
  * LayerNorm: biased variance, eps 1e-6, fp64, output rounded to bf16.
  * RoPE: inv_freq_i = theta**(-2i/36), i < 18; angles [row*f, col*f];
    rotate_half pairs (j, j+36); fp64, rounded to bf16.
  * attention: scale 1/sqrt(72), fp64 softmax, output rounded to bf16.
  * GELU: tanh form, evaluated as x / (1 + exp(-2u)) in fp64 (no cancellation),
    rounded to bf16 (blocks and mergers).
  * patch order: 2x2-block order for even grids (so the merger's 4
    neighbours are 4 consecutive rows), row-major otherwise.
  * merger: LayerNorm over the 4608 concatenated features, then
    fc1 -> GELU -> fc2, each GEMM FP8 block-128.
"""
from __future__ import annotations

import math

import numpy as np

from .numerics import E4M3_MAX, bf16_round, e4m3_decode, e4m3_encode

QBLK = 128                       # FP8 scaling block (1x128 activations, 128x128 weights)


# --------------------------------------------------------------------------
# FP8 block quantisation  [FRT s3; TRT recipe]
# --------------------------------------------------------------------------

def quant_act(y) -> tuple:
    """Per-row, per-128-column FP8 quantisation of bf16-valued activations
    [FRT s3: per-token / per-128-K-block activation quant; TRT recipe: scale amax / 448].

    Returns (codes uint8 [M, K], scales float32 [ceil(K/128), M]).
    """
    y = np.asarray(y, dtype=np.float64)
    M, K = y.shape
    nkb = -(-K // QBLK)
    codes = np.zeros((M, K), np.uint8)
    scales = np.zeros((nkb, M), np.float32)
    for g in range(nkb):
        blk = y[:, g * QBLK:(g + 1) * QBLK].astype(np.float32)   # exact: bf16 is a subset of fp32
        amax = np.max(np.abs(blk), axis=1)
        s = amax / np.float32(E4M3_MAX)                          # fp32 IEEE division
        safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
        v = blk / safe[:, None]                                  # fp32 IEEE division
        c = e4m3_encode(v)
        c[s == 0, :] = 0
        codes[:, g * QBLK:(g + 1) * QBLK] = c
        scales[g] = s
    return codes, scales


def quant_weight(w) -> tuple:
    """Per-128x128-block FP8 quantisation of a bf16-valued weight [N, K]
    [FRT introduction: block-128 W8A8 linears; TRT recipe: scale amax / 448].

    Returns (codes uint8 [N, K], scales float32 [ceil(N/128), ceil(K/128)]).
    """
    w = np.asarray(w, dtype=np.float64)
    N, K = w.shape
    nnb, nkb = -(-N // QBLK), -(-K // QBLK)
    codes = np.zeros((N, K), np.uint8)
    scales = np.zeros((nnb, nkb), np.float32)
    for i in range(nnb):
        for j in range(nkb):
            blk = w[i * QBLK:(i + 1) * QBLK, j * QBLK:(j + 1) * QBLK].astype(np.float32)
            amax = np.float32(np.max(np.abs(blk)))
            s = np.float32(amax / np.float32(E4M3_MAX))
            if s > 0:
                c = e4m3_encode(blk / s)
            else:
                c = np.zeros(blk.shape, np.uint8)
            codes[i * QBLK:(i + 1) * QBLK, j * QBLK:(j + 1) * QBLK] = c
            scales[i, j] = s
    return codes, scales


def dequant_act(codes, scales) -> np.ndarray:
    """Value represented by activation codes and their 1x128 scales (fp64) [FRT s3]."""
    M, K = codes.shape
    col_scale = np.repeat(scales.astype(np.float64), QBLK, axis=0)[:K].T   # [M, K]
    return e4m3_decode(codes) * col_scale


# --------------------------------------------------------------------------
# FP8 W8A8 block-scaled GEMM  [FRT s1, s3; VE vision_gemm_bias]
# --------------------------------------------------------------------------

def fp8_block_gemm(qa, sa, qw, sw, bias=None, residual=None) -> np.ndarray:
    """C[m, n] = bf16( sum_kb sa[kb, m] * sw[n // 128, kb] * P_kb[m, n] + bias[n] + residual[m, n] ).

    P_kb is the sum over the 128 columns of K block kb of decoded code
    products.  Each product is a multiple of 2**-18 below 2**18, so every
    partial sum of 128 of them is exact in fp64 whatever the order; the
    outer sum over K blocks is taken in fp64.  [FRT s1, s3: FP8 block-128 W8A8
    GEMMs with the bias (and residual) added in the same kernel; VE vision_gemm_bias.]
    """
    M, K = qa.shape
    N = qw.shape[0]
    a = e4m3_decode(qa)
    w = e4m3_decode(qw)
    nkb = -(-K // QBLK)
    acc = np.zeros((M, N), np.float64)
    wscale_cols = np.repeat(sw.astype(np.float64), QBLK, axis=0)[:N]       # [N, nkb]
    for kb in range(nkb):
        ks = slice(kb * QBLK, (kb + 1) * QBLK)
        part = a[:, ks] @ w[:, ks].T                                        # exact
        acc += (sa[kb].astype(np.float64)[:, None] * wscale_cols[:, kb][None, :]) * part
    if bias is not None:
        acc = acc + np.asarray(bias, np.float64)[None, :]
    if residual is not None:
        acc = acc + np.asarray(residual, np.float64)
    return bf16_round(acc)


def bf16_gemm(a, w, bias=None, residual=None) -> np.ndarray:
    """C[m, n] = bf16( sum_k a[m, k] w[n, k] + bias[n] + residual[m, n] ) for bf16 a, w.

    The bf16 linears of [FRT s4] (patch embedding, first three blocks,
    mergers) and [VE] dense_gemm_bf16 + vision_add_bias: the plain matrix
    product of the bf16 values, taken in fp64 (a library matmul as one step),
    then one bf16 rounding after the bias and residual adds.
    """
    acc = np.asarray(a, np.float64) @ np.asarray(w, np.float64).T
    if bias is not None:
        acc = acc + np.asarray(bias, np.float64)[None, :]
    if residual is not None:
        acc = acc + np.asarray(residual, np.float64)
    return bf16_round(acc)


# --------------------------------------------------------------------------
# LayerNorm and GELU  [FRT s3: LayerNorm and GELU(tanh) in the block chain; VE norm1_w/b]
# --------------------------------------------------------------------------

def layernorm_f64(x, gamma, beta, eps: float = 1e-6) -> np.ndarray:
    """Biased-variance LayerNorm in fp64, not rounded [FRT s3 block chain; VE norm1_w / norm1_b]."""
    x = np.asarray(x, np.float64)
    mu = x.mean(axis=1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * np.asarray(gamma, np.float64) + np.asarray(beta, np.float64)


def layernorm(x, gamma, beta, eps: float = 1e-6) -> np.ndarray:
    """LayerNorm rounded once to bf16, the block's normalised activation [FRT s3]."""
    return bf16_round(layernorm_f64(x, gamma, beta, eps))


def gelu_tanh_f64(x) -> np.ndarray:
    """GELU(tanh) = 0.5 x (1 + tanh(u)), u = sqrt(2/pi) (x + 0.044715 x^3), in fp64, not rounded
    [FRT s3: GELU(tanh)].

    Evaluated as x / (1 + exp(-2u)), which equals 0.5 x (1 + tanh(u)) exactly
    (1 + tanh(u) = 2 / (1 + exp(-2u))) but does not cancel for u << 0, where
    1 + tanh(u) in fp64 loses all its digits (u < -19, x < -5.6).
    """
    x = np.asarray(x, np.float64)
    u = math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-2.0 * u))


def gelu_tanh(x) -> np.ndarray:
    """GELU(tanh) rounded once to bf16 [FRT s3]."""
    return bf16_round(gelu_tanh_f64(x))


def ln_quant(x, gamma, beta, eps: float = 1e-6) -> tuple:
    """LayerNorm rounded to bf16, then 1x128 FP8 quant (the fused producer of [FRT s3])."""
    return quant_act(layernorm(x, gamma, beta, eps))


def gelu_quant(f) -> tuple:
    """GELU(tanh) rounded to bf16, then 1x128 FP8 quant (the fused producer of [FRT s3])."""
    return quant_act(gelu_tanh(f))


# --------------------------------------------------------------------------
# Patch order and 2D rotary embedding  [FRT s3: 2D rotary in rotate_half form; VE rope_inv_freq]
# --------------------------------------------------------------------------

def patch_positions(h: int, w: int) -> np.ndarray:
    """(row, col) of each patch of an h x w grid in token order, int64 [h*w, 2]
    [FRT s3: 2D positions for the rotary and the 2x2 merger; VE MergerLayer].

    Even grids use 2x2-block order: block (br, bc) in row-major order, and
    inside it (0,0), (0,1), (1,0), (1,1).  Odd grids use row-major order.
    """
    pos = []
    if h % 2 == 0 and w % 2 == 0:
        for br in range(h // 2):
            for bc in range(w // 2):
                for i in range(2):
                    for j in range(2):
                        pos.append((2 * br + i, 2 * bc + j))
    else:
        for r in range(h):
            for c in range(w):
                pos.append((r, c))
    return np.asarray(pos, dtype=np.int64).reshape(-1, 2)


def packed_positions(grids) -> tuple:
    """Positions of all packed images and their cu_seqlens [FRT s5: one attention window per image]."""
    pos = [patch_positions(h, w) for h, w in grids]
    cu = [0]
    for h, w in grids:
        cu.append(cu[-1] + h * w)
    return np.concatenate(pos, 0), np.asarray(cu, np.int64)


# --------------------------------------------------------------------------
# Patch embedding and interpolated position embedding
# [FRT s3: patch embedding, then the interpolated position table added; VE PATCH_DIM = 3*2*16*16 = 1536,
#  patch_embed_w [1152, 1536], pos_embed [2304, 1152], num_grid_per_side 48]
# --------------------------------------------------------------------------

POS_GRID = 48


def pos_embed_interp(table, h: int, w: int) -> np.ndarray:
    """Bilinear interpolation of the learned 48 x 48 position table to an h x w patch grid
    [FRT s3: interpolated pos_embed; VE num_grid_per_side 48].

    Sample points run from corner to corner: grid row r of h sits at table row
    r * 47 / (h - 1) (0 when h = 1), likewise for columns; each value mixes the
    four surrounding table entries with the usual bilinear weights.  fp64,
    not rounded: [h, w, C].
    """
    T = np.asarray(table, np.float64).reshape(POS_GRID, POS_GRID, -1)
    fy = np.arange(h, dtype=np.float64) * ((POS_GRID - 1) / (h - 1) if h > 1 else 0.0)
    fx = np.arange(w, dtype=np.float64) * ((POS_GRID - 1) / (w - 1) if w > 1 else 0.0)
    y0 = np.floor(fy).astype(np.int64)
    x0 = np.floor(fx).astype(np.int64)
    y1 = np.minimum(y0 + 1, POS_GRID - 1)
    x1 = np.minimum(x0 + 1, POS_GRID - 1)
    dy = (fy - y0)[:, None, None]
    dx = (fx - x0)[None, :, None]
    return ((1 - dy) * (1 - dx) * T[y0][:, x0] + (1 - dy) * dx * T[y0][:, x1]
            + dy * (1 - dx) * T[y1][:, x0] + dy * dx * T[y1][:, x1])


def patch_embed(pixels, w, b, table, grids) -> np.ndarray:
    """x = bf16( pixels @ w^T + b + pos ) over packed images in token order, where pos is
    the interpolated position embedding of each patch rounded to bf16.

    pixels: [n, 1536] patch rows (already normalised and patchified); w [1152, 1536].
    [FRT s3: patch_embed then the interpolated pos_embed; VE PATCH_DIM 1536.]
    """
    pos = []
    for h, wd in grids:
        grid = pos_embed_interp(table, h, wd)
        rc = patch_positions(h, wd)
        pos.append(grid[rc[:, 0], rc[:, 1]])
    return bf16_gemm(pixels, w, bias=b, residual=bf16_round(np.concatenate(pos, 0)))


def rope_inv_freq(head_dim: int = 72, theta: float = 10000.0) -> np.ndarray:
    """head_dim/4 frequencies theta**(-2i/(head_dim/2)), fp64 [VE rope_inv_freq; FRT s3 2D RoPE]."""
    half = head_dim // 2
    i = np.arange(half // 2, dtype=np.float64)
    return theta ** (-2.0 * i / half)


def rope_angles(pos, head_dim: int = 72, theta: float = 10000.0) -> np.ndarray:
    """Rotation angle of pair j (0 <= j < head_dim/2): row*f_j for the first
    head_dim/4 pairs, col*f_(j - head_dim/4) for the rest.  fp64 [n, head_dim/2].
    [FRT s3: 2D RoPE; VE rope_inv_freq.]"""
    f = rope_inv_freq(head_dim, theta)
    pos = np.asarray(pos, np.float64)
    return np.concatenate([pos[:, :1] * f[None, :], pos[:, 1:2] * f[None, :]], axis=1)


def rope_rotate(x, angles) -> np.ndarray:
    """rotate_half rotary on the last axis of x [n, ..., d]; pairs (j, j + d/2) [FRT s3].

    x'_j = x_j cos a_j - x_(j+d/2) sin a_j,  x'_(j+d/2) = x_(j+d/2) cos a_j + x_j sin a_j.
    fp64, not rounded.  angles is [n, d/2] and broadcasts over middle axes.
    """
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    h = d // 2
    shape = (angles.shape[0],) + (1,) * (x.ndim - 2) + (h,)
    c = np.cos(angles).reshape(shape)
    s = np.sin(angles).reshape(shape)
    x1, x2 = x[..., :h], x[..., h:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def apply_rope_qkv(qkv, pos, heads: int = 16, head_dim: int = 72, theta: float = 10000.0) -> np.ndarray:
    """Rotate the q and k parts of a packed qkv [n, 3*heads*head_dim] ([n, 3, heads, head_dim]
    order); v is unchanged.  Result rounded to bf16.  [FRT s3: RoPE on q and k after
    the QKV projection.]"""
    qkv = np.asarray(qkv, np.float64)
    n = qkv.shape[0]
    t = qkv.reshape(n, 3, heads, head_dim)
    ang = rope_angles(pos, head_dim, theta)
    out = t.copy()
    out[:, 0] = rope_rotate(t[:, 0], ang)
    out[:, 1] = rope_rotate(t[:, 1], ang)
    return bf16_round(out.reshape(n, -1))


# --------------------------------------------------------------------------
# Block-diagonal non-causal attention  [FRT s1, s3: full bidirectional flash attention; s5 cu_seqlens]
# --------------------------------------------------------------------------

def attention_varlen(qkv, cu_seqlens, heads: int = 16, head_dim: int = 72, scale=None) -> np.ndarray:
    """softmax(q k^T * scale) v per segment and head, fp64; output [n, heads*head_dim] rounded to bf16
    [FRT s3: full bidirectional attention; s5: cu_seqlens segments]."""
    qkv = np.asarray(qkv, np.float64)
    n = qkv.shape[0]
    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    t = qkv.reshape(n, 3, heads, head_dim)
    out = np.zeros((n, heads, head_dim), np.float64)
    cu = [int(c) for c in cu_seqlens]
    for a, b in zip(cu[:-1], cu[1:]):
        if b <= a:
            continue
        for h in range(heads):
            q, k, v = t[a:b, 0, h], t[a:b, 1, h], t[a:b, 2, h]
            s = (q @ k.T) * scale
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p = p / p.sum(axis=1, keepdims=True)
            out[a:b, h] = p @ v
    return bf16_round(out.reshape(n, heads * head_dim))


# --------------------------------------------------------------------------
# Block, merger, tower  [FRT s3; VE ViTBlock / MergerLayer / VisionEncoder]
# --------------------------------------------------------------------------

def quantize_block_weights(p: dict) -> dict:
    """FP8 codes + 128x128 scales of the four linear layers of a block (bf16-valued inputs)
    [FRT introduction: block-128 W8A8]."""
    q = dict(p)
    for name in ("qkv", "proj", "fc1", "fc2"):
        q[name + "_q"], q[name + "_s"] = quant_weight(p[name + "_w"])
    return q


def quantize_merger_weights(p: dict) -> dict:
    """FP8 codes + 128x128 scales of the merger's fc1 and fc2 [FRT introduction, s3 merger]."""
    q = dict(p)
    for name in ("fc1", "fc2"):
        q[name + "_q"], q[name + "_s"] = quant_weight(p[name + "_w"])
    return q


def block_forward(x, w: dict, cu_seqlens, pos, eps: float = 1e-6, keep: bool = False):
    """One ViT block.  x is bf16-valued [n, 1152]; w holds bf16-valued LN/bias vectors and
    the FP8 codes/scales of the linears (see quantize_block_weights).

    Returns x2, or (x2, dict of every intermediate) with keep=True.
    [FRT s3: the per-block chain LN -> QKV -> RoPE -> attention -> proj + residual ->
    LN -> fc1 -> GELU -> fc2 + residual; VE ViTBlock.]
    """
    x = np.asarray(x, np.float64)
    st = {}
    st["q1"], st["s1"] = ln_quant(x, w["norm1_w"], w["norm1_b"], eps)
    st["qkv"] = fp8_block_gemm(st["q1"], st["s1"], w["qkv_q"], w["qkv_s"], bias=w["qkv_b"])
    st["qkv_rot"] = apply_rope_qkv(st["qkv"], pos)
    st["attn"] = attention_varlen(st["qkv_rot"], cu_seqlens)
    st["qo"], st["so"] = quant_act(st["attn"])
    st["x1"] = fp8_block_gemm(st["qo"], st["so"], w["proj_q"], w["proj_s"], bias=w["proj_b"], residual=x)
    st["q2"], st["s2"] = ln_quant(st["x1"], w["norm2_w"], w["norm2_b"], eps)
    st["f"] = fp8_block_gemm(st["q2"], st["s2"], w["fc1_q"], w["fc1_s"], bias=w["fc1_b"])
    st["qg"], st["sg"] = gelu_quant(st["f"])
    st["x2"] = fp8_block_gemm(st["qg"], st["sg"], w["fc2_q"], w["fc2_s"], bias=w["fc2_b"], residual=st["x1"])
    return (st["x2"], st) if keep else st["x2"]


def block_forward_bf16(x, w: dict, cu_seqlens, pos, eps: float = 1e-6, keep: bool = False):
    """One ViT block with bf16 linears [FRT s4: the first three blocks stay bf16]: LayerNorm and
    GELU outputs rounded to bf16 and fed to bf16 GEMMs (no FP8 quantisation); w holds the
    bf16-valued weights of block_params (qkv_w, proj_w, fc1_w, fc2_w [out, in]).
    """
    x = np.asarray(x, np.float64)
    st = {}
    st["h1"] = layernorm(x, w["norm1_w"], w["norm1_b"], eps)
    st["qkv"] = bf16_gemm(st["h1"], w["qkv_w"], bias=w["qkv_b"])
    st["qkv_rot"] = apply_rope_qkv(st["qkv"], pos)
    st["attn"] = attention_varlen(st["qkv_rot"], cu_seqlens)
    st["x1"] = bf16_gemm(st["attn"], w["proj_w"], bias=w["proj_b"], residual=x)
    st["h2"] = layernorm(st["x1"], w["norm2_w"], w["norm2_b"], eps)
    st["f"] = bf16_gemm(st["h2"], w["fc1_w"], bias=w["fc1_b"])
    st["g"] = gelu_tanh(st["f"])
    st["x2"] = bf16_gemm(st["g"], w["fc2_w"], bias=w["fc2_b"], residual=st["x1"])
    return (st["x2"], st) if keep else st["x2"]


def merger_forward_bf16(x, w: dict, eps: float = 1e-6, keep: bool = False):
    """2x2 merger with bf16 linears [FRT s4: the mergers stay bf16]."""
    x = np.asarray(x, np.float64)
    n, c = x.shape
    st = {}
    st["h1"] = layernorm(x.reshape(n // 4, 4 * c), w["norm_w"], w["norm_b"], eps)
    st["h"] = bf16_gemm(st["h1"], w["fc1_w"], bias=w["fc1_b"])
    st["g"] = gelu_tanh(st["h"])
    st["out"] = bf16_gemm(st["g"], w["fc2_w"], bias=w["fc2_b"])
    return (st["out"], st) if keep else st["out"]


def merger_forward(x, w: dict, eps: float = 1e-6, keep: bool = False):
    """2x2 merger: 4 consecutive rows -> one 4608 row, LayerNorm, fc1, GELU, fc2
    [FRT s3: 2x2 merger on the DeepStack taps; VE MergerLayer]."""
    x = np.asarray(x, np.float64)
    n, c = x.shape
    xm = x.reshape(n // 4, 4 * c)
    st = {}
    st["q1"], st["s1"] = ln_quant(xm, w["norm_w"], w["norm_b"], eps)
    st["h"] = fp8_block_gemm(st["q1"], st["s1"], w["fc1_q"], w["fc1_s"], bias=w["fc1_b"])
    st["qg"], st["sg"] = gelu_quant(st["h"])
    st["out"] = fp8_block_gemm(st["qg"], st["sg"], w["fc2_q"], w["fc2_s"], bias=w["fc2_b"])
    return (st["out"], st) if keep else st["out"]


def tower_forward(x, blocks, mergers, grids, taps_after=(8, 16, 24, 27), eps: float = 1e-6,
                  on_block=None):
    """27 blocks over packed images, a merger after each tapped block.

    blocks: list of block weight dicts, each either quantised (quantize_block_weights: FP8
    block) or the bf16 weights themselves (no "qkv_q": bf16 block); mergers likewise.
    Returns the list of merger outputs (one per tap).
    [FRT s3: DeepStack taps after blocks 8, 16, 24 and the final merger; VE VisionEncoder
    deepstack indexes.]
    """
    pos, cu = packed_positions(grids)
    h = np.asarray(x, np.float64)
    taps = []
    for b, w in enumerate(blocks, start=1):
        h = (block_forward if "qkv_q" in w else block_forward_bf16)(h, w, cu, pos, eps)
        if on_block is not None:
            on_block(b, h)
        if b in taps_after:
            m = mergers[taps_after.index(b)]
            taps.append((merger_forward if "fc1_q" in m else merger_forward_bf16)(h, m, eps))
    return taps
