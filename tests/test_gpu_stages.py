"""GPU parity of each stage against the CPU oracle, through the C ABI.

Every CUDA stage is fed the oracle's own inputs for that stage (seeded
synthetic tensors from workloads.py).  FP8 codes and scales are compared
bit for bit; bf16 stage outputs within rel-L2 <= 1e-2 and max-abs <= 3e-2
(the stated per-stage tolerance).  Shapes cover several 128-tiles, ragged
M / N / K tails, one-row and one-token cases, and the full 6256-patch sizes.
"""
import math

import numpy as np
import pytest
import torch

from oracle import numerics as onum
from oracle import vit as ov
from quantized_vit_encoder_b200 import workloads as wl

pytestmark = pytest.mark.gpu

REL_L2, MAX_ABS = 1e-2, 3e-2


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def rel_l2(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def bf16_ulp(v):
    """Spacing of bf16 values at |v| (2^(e-7) for |v| in [2^e, 2^(e+1)))."""
    v = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(v, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def assert_close(got, want, rel=REL_L2, mabs=MAX_ABS, what=""):
    """rel-L2 <= rel, and every element within max(mabs, one bf16 ulp of the reference):
    a bf16 output cannot be closer than one rounding step, which exceeds 3e-2 for |v| >= 4."""
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), what
    r = rel_l2(got, want)
    d = np.abs(got - want)
    m = float(d.max()) if got.size else 0.0
    worst = float((d / np.maximum(mabs, bf16_ulp(want))).max()) if got.size else 0.0
    assert r <= rel and worst <= 1.0, f"{what}: rel_l2={r:.3e} max_abs={m:.3e} (worst/allowed {worst:.2f})"
    return r, m


def assert_codes_equal(q_gpu, s_gpu, q_ref, s_ref, what=""):
    M = q_ref.shape[0]
    qg = q_gpu.cpu().numpy()
    sg = s_gpu.cpu().numpy()[:, :M]
    bad_s = np.argwhere(sg != s_ref)
    assert bad_s.size == 0, f"{what}: {len(bad_s)} scales differ, first {bad_s[:3].tolist()}"
    bad_q = np.argwhere(qg != q_ref)
    assert bad_q.size == 0, f"{what}: {len(bad_q)} codes differ, first {bad_q[:3].tolist()}"


def bf16(shape, seed, std=1.0):
    return wl.random_bf16(shape, seed, std)


# ----------------------------------------------------------------- quantisation

@pytest.mark.parametrize("M,K", [(1, 16), (127, 1152), (129, 4304), (300, 4608), (972, 1152), (6256, 1152)])
def test_quant_act_bit_exact(lib, M, K):
    from quantized_vit_encoder_b200 import vitq
    x = bf16((M, K), 10 + M + K, 3.0)
    q, s = vitq.quant_act(x.cuda())
    qr, sr = ov.quant_act(f64(x))
    assert_codes_equal(q, s, qr, sr, f"quant_act {M}x{K}")


def test_quant_act_every_bf16_value(lib):
    """All 65536 bf16 bit patterns (finite ones), in groups with different amax, encode bit-exactly."""
    from quantized_vit_encoder_b200 import vitq
    bits = np.arange(65536, dtype=np.uint32)
    vals = onum.bf16_bits_to_f64(bits)
    vals = vals[np.isfinite(vals)]
    vals = vals[np.abs(vals) < 1e30]               # keep amax/448 and v/s finite in fp32
    g = np.random.default_rng(0)
    rows = []
    for amax in (1.0, 448.0, 3.0e-3, 7.5e4, 1e-30):
        v = vals[np.abs(vals) <= amax]
        v = g.permutation(v)
        pad = (-len(v)) % 127
        v = np.concatenate([v, np.zeros(pad)]).reshape(-1, 127)
        rows.append(np.concatenate([v, np.full((v.shape[0], 1), amax)], 1))
    x = np.concatenate(rows, 0)
    xt = torch.from_numpy(x).to(torch.bfloat16)
    q, s = vitq.quant_act(xt.cuda())
    qr, sr = ov.quant_act(f64(xt))
    assert_codes_equal(q, s, qr, sr, "exhaustive")


@pytest.mark.parametrize("N,K", [(3456, 1152), (1152, 4304), (4304, 1152), (200, 272)])
def test_quant_weight_bit_exact(lib, N, K):
    from quantized_vit_encoder_b200 import vitq
    w = bf16((N, K), 20 + N, 0.02)
    q, s = vitq.quant_weight(w.cuda())
    qr, sr = ov.quant_weight(f64(w))
    assert np.array_equal(s.cpu().numpy(), sr)
    assert np.array_equal(q.cpu().numpy(), qr)


@pytest.mark.parametrize("M,K,scale", [(1, 1152, 1.0), (129, 1152, 10.0), (972, 1152, 0.1), (301, 4608, 1.0),
                                       (6256, 1152, 1.0)])
def test_ln_quant_bit_exact(lib, M, K, scale):
    from quantized_vit_encoder_b200 import vitq
    x = bf16((M, K), 30 + M, scale)
    g = (1 + wl.random_bf16((K,), 31, 0.02).float()).to(torch.bfloat16)
    b = wl.random_bf16((K,), 32, 0.01)
    q, s = vitq.ln_quant(x.cuda(), g.cuda(), b.cuda())
    qr, sr = ov.ln_quant(f64(x), f64(g), f64(b), 1e-6)
    assert_codes_equal(q, s, qr, sr, f"ln_quant {M}x{K}")


@pytest.mark.parametrize("M,K", [(1, 4304), (129, 4304), (972, 4304), (100, 4608), (6256, 4304)])
def test_gelu_quant_bit_exact(lib, M, K):
    from quantized_vit_encoder_b200 import vitq
    f = bf16((M, K), 40 + M, 1.5)
    q, s = vitq.gelu_quant(f.cuda())
    qr, sr = ov.gelu_quant(f64(f))
    assert_codes_equal(q, s, qr, sr, f"gelu_quant {M}x{K}")


def test_gelu_quant_wide_range_bands(lib):
    """Rows of narrow x bands covering [-12, 9]: every group's scale follows its band, so the
    codes see the bf16 GELU values everywhere, including the far negative tail."""
    from quantized_vit_encoder_b200 import vitq
    rows = 420
    lo = torch.linspace(-12.0, 9.0, rows + 1)[:-1]
    g = torch.Generator().manual_seed(45)
    f = (lo[:, None] + torch.rand((rows, 256), generator=g) * 0.05).to(torch.bfloat16)
    q, s = vitq.gelu_quant(f.cuda())
    qr, sr = ov.gelu_quant(f64(f))
    assert_codes_equal(q, s, qr, sr, "gelu wide")


def test_gelu_quant_every_bf16_value(lib):
    """All 65024 finite bf16 bit patterns, in pattern order (each group of 128 holds
    neighbouring values of one sign), through GELU + quant against the oracle."""
    from quantized_vit_encoder_b200 import vitq
    pats = np.arange(65536, dtype=np.uint32)
    pats = pats[((pats >> 7) & 0xFF) != 0xFF]                       # drop inf / NaN
    f = torch.from_numpy((pats << 16).view(np.float32)).to(torch.bfloat16).reshape(-1, 256)
    q, s = vitq.gelu_quant(f.cuda())
    qr, sr = ov.gelu_quant(f64(f))
    assert_codes_equal(q, s, qr, sr, "gelu every bf16")


def test_ln_quant_offset_mean(lib):
    """Rows with |mean| several times their spread (the one-pass variance is still exact enough)."""
    from quantized_vit_encoder_b200 import vitq
    M, K = 257, 1152
    x = (wl.random_bf16((M, K), 46, 1.0).float() + torch.linspace(-8, 8, M)[:, None]).to(torch.bfloat16)
    g = (1 + wl.random_bf16((K,), 47, 0.02).float()).to(torch.bfloat16)
    b = wl.random_bf16((K,), 48, 0.01)
    q, s = vitq.ln_quant(x.cuda(), g.cuda(), b.cuda())
    qr, sr = ov.ln_quant(f64(x), f64(g), f64(b), 1e-6)
    assert_codes_equal(q, s, qr, sr, "ln offset")


# ----------------------------------------------------------------- GEMM

GEMM_SHAPES = [
    (1, 128, 128), (128, 128, 1152), (129, 3456, 1152), (256, 1152, 4304), (972, 4304, 1152),
    (300, 2048, 4608), (77, 136, 272), (6256, 1152, 1152),
]


@pytest.mark.parametrize("pair", [0, 1], ids=["cta", "pair"])
@pytest.mark.parametrize("bn", [64, 128, 256])
@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_fp8_gemm_matches_oracle(lib, monkeypatch, pair, bn, M, N, K):
    """One CTA per tile and CTA pairs (cta_group::2 MMA over 256-row tiles; pairs run
    64-wide requests as 128)."""
    from quantized_vit_encoder_b200 import vitq
    monkeypatch.setenv("VITQ_GEMM_BN", str(bn))
    monkeypatch.setenv("VITQ_GEMM_PAIR", str(pair))
    a = bf16((M, K), 50 + M, 1.0)
    w = bf16((N, K), 51 + N, 0.02)
    bias = bf16((N,), 52, 0.01)
    res = bf16((M, N), 53, 1.0)
    qa, sa = ov.quant_act(f64(a))
    qw, sw = ov.quant_weight(f64(w))
    ref = ov.fp8_block_gemm(qa, sa, qw, sw, f64(bias), f64(res))
    lds = (M + 3) // 4 * 4
    sa_pad = np.zeros((sa.shape[0], lds), np.float32)
    sa_pad[:, :M] = sa
    dev = "cuda"
    out = vitq.fp8_block_gemm(torch.from_numpy(qa).to(dev), torch.from_numpy(sa_pad).to(dev),
                              torch.from_numpy(qw).to(dev), torch.from_numpy(sw).to(dev),
                              bias.to(dev), res.to(dev))
    got = f64(out)
    assert_close(got, ref, what=f"gemm {M}x{N}x{K} bn{bn} pair{pair}")
    # the promotion is fp32 against an fp64 oracle: nearly every bf16 output is identical
    assert np.mean(got == ref) > 0.97


@pytest.mark.parametrize("M,N,K,res", [(256, 3456, 1152, False), (300, 1152, 4304, True),
                                       (972, 4304, 1152, False), (6256, 1152, 1152, True)])
def test_fp8_gemm_tile_width_invariant(lib, monkeypatch, M, N, K, res):
    """Every tile width gives the same bits: each output element is the same chain of
    per-K-block FMAs whatever the tile, so the library may pick the width from M (more,
    narrower tiles for small M) without making a packed batch differ from its images."""
    from quantized_vit_encoder_b200 import vitq
    a = bf16((M, K), 80 + M, 1.0)
    w = bf16((N, K), 81 + N, 0.02)
    bias = bf16((N,), 82, 0.01).cuda()
    r = bf16((M, N), 83, 1.0).cuda() if res else None
    qa, sa = vitq.quant_act(a.cuda())
    qw, sw = vitq.quant_weight(w.cuda())
    outs = []
    for bn in (64, 128, 256):
        monkeypatch.setenv("VITQ_GEMM_BN", str(bn))
        outs.append(vitq.fp8_block_gemm(qa, sa, qw, sw, bias, r).view(torch.int16).cpu())
    monkeypatch.delenv("VITQ_GEMM_BN")
    outs.append(vitq.fp8_block_gemm(qa, sa, qw, sw, bias, r).view(torch.int16).cpu())   # the library's pick
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


BF16_GEMM_SHAPES = [
    (1, 128, 64), (128, 1152, 1536), (129, 3456, 1152), (300, 4304, 1152), (972, 1152, 4304),
    (77, 136, 72), (6256, 1152, 1536),
]


@pytest.mark.parametrize("bn", [128, 256])
@pytest.mark.parametrize("M,N,K", BF16_GEMM_SHAPES)
def test_bf16_gemm_matches_oracle(lib, monkeypatch, bn, M, N, K):
    """fp32 accumulation over all of K in TMEM against the fp64 oracle (ragged M, N and K tails)."""
    from quantized_vit_encoder_b200 import vitq
    monkeypatch.setenv("VITQ_GEMM_BN", str(bn))
    a = bf16((M, K), 70 + M, 1.0)
    w = bf16((N, K), 71 + N, 0.03)
    bias = bf16((N,), 72, 0.01)
    res = bf16((M, N), 73, 1.0)
    ref = ov.bf16_gemm(f64(a), f64(w), f64(bias), f64(res))
    got = f64(vitq.bf16_gemm(a.cuda(), w.cuda(), bias.cuda(), res.cuda()))
    assert_close(got, ref, what=f"bf16 gemm {M}x{N}x{K} bn{bn}")
    assert np.mean(got == ref) > 0.97
    plain = f64(vitq.bf16_gemm(a.cuda(), w.cuda()))
    assert_close(plain, ov.bf16_gemm(f64(a), f64(w)), what="bf16 gemm plain")


def test_fp8_gemm_no_bias_no_residual(lib):
    from quantized_vit_encoder_b200 import vitq
    M, N, K = 200, 384, 640
    a, w = bf16((M, K), 60, 2.0), bf16((N, K), 61, 0.05)
    qa, sa = ov.quant_act(f64(a))
    qw, sw = ov.quant_weight(f64(w))
    ref = ov.fp8_block_gemm(qa, sa, qw, sw)
    out = vitq.fp8_block_gemm(torch.from_numpy(qa).cuda(), torch.from_numpy(sa).cuda(),
                              torch.from_numpy(qw).cuda(), torch.from_numpy(sw).cuda())
    assert_close(f64(out), ref, what="gemm plain")


# ----------------------------------------------------------------- positions and RoPE

def test_positions_match_oracle(lib):
    from quantized_vit_encoder_b200 import vitq
    grids = [(54, 18), (46, 136), (24, 38), (32, 32), (36, 27), (1, 1)]
    pos, cu = vitq.positions(grids)
    pr, cr = ov.packed_positions(grids)
    assert np.array_equal(pos.cpu().numpy(), pr)
    assert np.array_equal(cu.cpu().numpy(), cr)


def test_rope_table_and_apply(lib):
    from quantized_vit_encoder_b200 import vitq
    grids = [(46, 136), (36, 27)]
    pos, _ = vitq.positions(grids)
    cs = vitq.rope_table(pos)
    pr, _ = ov.packed_positions(grids)
    ang = ov.rope_angles(pr)
    assert np.max(np.abs(cs.cpu().numpy()[:, :36] - np.cos(ang))) < 1e-6
    assert np.max(np.abs(cs.cpu().numpy()[:, 36:] - np.sin(ang))) < 1e-6
    n = pr.shape[0]
    qkv = bf16((n, 3456), 70, 1.0)
    got = vitq.rope2d_(qkv.cuda().clone(), cs)
    ref = ov.apply_rope_qkv(f64(qkv), pr)
    assert_close(f64(got), ref, what="rope")
    assert np.array_equal(f64(got)[:, 2304:], f64(qkv)[:, 2304:])       # v untouched
    # with VITQ_V_FP16 the q, k results are identical and v becomes its round-to-nearest
    # fp16 value: exact for 2^-14 <= |v| < 65504, within 2^-25 below (fp16 subnormals)
    got16 = vitq.rope2d_(qkv.cuda().clone(), cs, flags=vitq.V_FP16)
    assert torch.equal(got16[:, :2304], got[:, :2304])
    v16 = got16[:, 2304:].contiguous().view(torch.float16).float().cpu().double().numpy()
    v = f64(qkv)[:, 2304:]
    assert np.array_equal(v16, qkv[:, 2304:].float().half().double().numpy())     # torch's RN cast
    normal = np.abs(v) >= 2.0 ** -14
    assert np.array_equal(v16[normal], v[normal]) and np.all(np.abs(v16 - v) <= 2.0 ** -25)


def test_rope_v_fp16_range_guard(lib):
    """v beyond the fp16 range: clamped to +-65504, NaN kept, and the device error word
    reports VITQ_ERR_RANGE once (the read clears it); values in range are untouched."""
    from quantized_vit_encoder_b200 import vitq
    pos, _ = vitq.positions([(2, 4)])
    cs = vitq.rope_table(pos)
    qkv = bf16((8, 3456), 71, 1.0)
    qkv[3, 2304 + 5] = 1.0e5
    qkv[3, 2304 + 6] = -3.0e38
    qkv[5, 2304 + 100] = float("nan")
    qkv[6, 2304 + 7] = 65536.0        # bf16 has no 65504: the nearest values are 65280 and 65536
    qkv[6, 2304 + 8] = 65280.0        # in range: kept exactly
    assert vitq.device_error() == vitq.OK
    got = vitq.rope2d_(qkv.cuda().clone(), cs, flags=vitq.V_FP16)
    assert vitq.device_error() == vitq.ERR_RANGE
    assert vitq.device_error() == vitq.OK
    v16 = got[:, 2304:].contiguous().view(torch.float16).float().cpu()
    v = qkv[:, 2304:].float()
    assert v16[3, 5] == 65504.0 and v16[3, 6] == -65504.0 and v16[6, 7] == 65504.0 and v16[6, 8] == 65280.0
    assert torch.isnan(v16[5, 100])
    keep = torch.ones_like(v, dtype=torch.bool)
    keep[3, 5] = keep[3, 6] = keep[5, 100] = keep[6, 7] = False
    assert torch.equal(v16[keep], v.half().float()[keep])
    # no flag when everything fits
    vitq.rope2d_(bf16((8, 3456), 72, 1.0).cuda(), cs, flags=vitq.V_FP16)
    assert vitq.device_error() == vitq.OK


# ----------------------------------------------------------------- attention

ATTN_CASES = [
    [1], [127], [128], [129], [256], [300, 1, 77, 128], [972], [972, 6256, 912, 1024],
]


def _v_to_f16(qkv_dev):
    """v part converted to fp16 in place (exact), as the block does before attention."""
    t = qkv_dev.clone()
    t[:, 2304:] = t[:, 2304:].float().half().view(torch.bfloat16)
    return t


@pytest.mark.parametrize("v16", [False, True], ids=["bf16v", "f16v"])
@pytest.mark.parametrize("lens", ATTN_CASES, ids=lambda v: "-".join(map(str, v)))
def test_attention_matches_oracle(lib, lens, v16):
    from quantized_vit_encoder_b200 import vitq
    n = sum(lens)
    cu = wl.random_cu_seqlens(lens)
    qkv = bf16((n, 3456), 80 + n, 1.0)
    ref = ov.attention_varlen(f64(qkv), cu)
    dq = _v_to_f16(qkv.cuda()) if v16 else qkv.cuda()
    got = vitq.attention_varlen(dq, torch.tensor(cu, dtype=torch.int32, device="cuda"), max(lens),
                                flags=vitq.V_FP16 if v16 else 0)
    r, _ = assert_close(f64(got), ref, what=f"attention {lens}")
    if v16 and n >= 128:
        # fp16 P: the only remaining difference is the final bf16 rounding of O
        assert r < 1.5e-3, r


def test_attention_large_logits_rescale(lib):
    """Scores spanning a wide range force the running-max rescale path."""
    from quantized_vit_encoder_b200 import vitq
    n = 700
    g = torch.Generator().manual_seed(90)
    qkv = torch.randn((n, 3456), generator=g)
    qkv[:, :2304] *= torch.linspace(0.2, 4.0, n)[:, None]          # growing norms along the sequence
    qkv = qkv.to(torch.bfloat16)
    ref = ov.attention_varlen(f64(qkv), [0, n])
    got = vitq.attention_varlen(qkv.cuda(), torch.tensor([0, n], dtype=torch.int32, device="cuda"), n)
    assert_close(f64(got), ref, what="attention rescale")


def test_attention_full_6256_sampled_rows(lib):
    """Full 46x136 image: compare 256 sampled query rows of every head against the oracle."""
    from quantized_vit_encoder_b200 import vitq
    n = 6256
    qkv = bf16((n, 3456), 95, 1.0)
    got = f64(vitq.attention_varlen(qkv.cuda(), torch.tensor([0, n], dtype=torch.int32, device="cuda"), n))
    rows = np.random.default_rng(1).choice(n, 256, replace=False)
    t = f64(qkv).reshape(n, 3, 16, 72)
    ref = np.zeros((256, 16, 72))
    for h in range(16):
        s = t[rows, 0, h] @ t[:, 1, h].T / math.sqrt(72)
        s -= s.max(1, keepdims=True)
        p = np.exp(s)
        ref[:, h] = (p / p.sum(1, keepdims=True)) @ t[:, 2, h]
    assert_close(got[rows], onum.bf16_round(ref.reshape(256, -1)), what="attention 6256 sampled")


def test_zero_rows_are_no_ops(lib):
    """Zero rows through every stage entry point: status ok, outputs untouched, no device error."""
    from quantized_vit_encoder_b200 import vitq
    L = vitq.load()
    s = vitq._stream(None)
    p = vitq._p
    x = torch.full((4, 1152), 1.5, dtype=torch.bfloat16, device="cuda")
    f = torch.full((4, 4304), 1.5, dtype=torch.bfloat16, device="cuda")
    q = torch.full((4, 4304), 7, dtype=torch.uint8, device="cuda")
    sc = torch.full((34, 4), -1.0, dtype=torch.float32, device="cuda")
    g = torch.ones(1152, dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(1152, dtype=torch.bfloat16, device="cuda")
    w = torch.full((1152, 1152), 3, dtype=torch.uint8, device="cuda")
    sw = torch.ones((9, 9), dtype=torch.float32, device="cuda")
    out = torch.full((4, 1152), 2.0, dtype=torch.bfloat16, device="cuda")
    assert L.vit_quant_act(p(x), 0, 1152, 1152, p(q), p(sc), 4, s) == 0
    assert L.vit_ln_quant(p(x), 0, 1152, 1152, p(g), p(b), 1e-6, p(q), p(sc), 4, s) == 0
    assert L.vit_gelu_quant(p(f), 0, 4304, 4304, p(q), p(sc), 4, s) == 0
    assert L.fp8_block_gemm(p(q), p(sc), 4, p(w), p(sw), None, None, p(out), 0, 1152, 1152, s) == 0
    cu0 = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert L.vit_attention_varlen(p(f), 0, p(cu0), 0, 0, 0.1, 0, p(out), s) == 0
    torch.cuda.synchronize()
    assert vitq.device_error() == 0
    assert torch.all(q == 7) and torch.all(sc == -1.0) and torch.all(out == 2.0)


def test_attention_empty_segment_in_a_packed_batch(lib):
    """A zero-length segment between two others: its CTAs do nothing, the others are unaffected."""
    from quantized_vit_encoder_b200 import vitq
    lens = [5, 0, 7]
    n = sum(lens)
    cu = wl.random_cu_seqlens(lens)
    qkv = bf16((n, 3456), 77, 1.0)
    ref = ov.attention_varlen(f64(qkv), cu)
    got = vitq.attention_varlen(qkv.cuda(), torch.tensor(cu, dtype=torch.int32, device="cuda"), max(lens))
    torch.cuda.synchronize()
    assert vitq.device_error() == 0
    assert_close(f64(got), ref, what="attention with an empty segment")
