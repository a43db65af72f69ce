"""Pins of the CPU oracle against things other than itself.

Each test ties one oracle function to a closed form, an exhaustive table, a
library routine (torch casts), a brute-force loop on a tiny case, or an
invariant, so that a dropped term, a wrong sign or index, or a transposed
operand in the oracle fails here.
"""
import math

import numpy as np
import pytest
import torch

from oracle import numerics as nm
from oracle import vit as ov

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ---------------------------------------------------------------- bf16

def test_bf16_round_matches_torch_cast():
    g = torch.Generator().manual_seed(1)
    x = torch.randn(200000, generator=g) * torch.exp(torch.randn(200000, generator=g) * 6)
    ref = x.to(torch.bfloat16).to(torch.float64).numpy()
    got = nm.bf16_round(x.to(torch.float64).numpy())
    assert np.array_equal(ref, got)


def test_bf16_round_ties_to_even():
    # 1 + 2**-8 lies halfway between 1 and 1 + 2**-7: ties go to the even mantissa (1.0).
    assert nm.bf16_round(1.0 + 2.0 ** -8) == 1.0
    # 1 + 3 * 2**-8 lies halfway between 1 + 2**-7 and 1 + 2**-6: goes up to the even one.
    assert nm.bf16_round(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    # fp64 values just off a tie are not double-rounded.
    assert nm.bf16_round(1.0 + 2.0 ** -8 + 2.0 ** -40) == 1.0 + 2.0 ** -7


def test_bf16_bits_roundtrip():
    bits = np.arange(0, 65536, dtype=np.uint32)
    vals = nm.bf16_bits_to_f64(bits)
    finite = np.isfinite(vals)
    assert np.array_equal(nm.bf16_round(vals[finite]), vals[finite])
    ref = torch.from_numpy(bits.astype(np.int32)).to(torch.int16).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ref), np.isnan(vals))
    assert np.array_equal(ref[~np.isnan(ref)], vals[~np.isnan(vals)])


# ---------------------------------------------------------------- E4M3

def test_e4m3_decode_closed_form_points():
    d = nm.e4m3_decode(np.arange(256))
    assert d[0x7E] == 448.0 and d[0xFE] == -448.0          # largest finite
    assert d[0x08] == 2.0 ** -6                             # smallest normal
    assert d[0x01] == 2.0 ** -9                             # smallest subnormal
    assert d[0x07] == 7 * 2.0 ** -9                         # largest subnormal
    assert d[0x38] == 1.0 and d[0x40] == 2.0                # exponent bias 7
    assert d[0x39] == 1.125                                 # 3 mantissa bits
    assert np.isnan(d[0x7F]) and np.isnan(d[0xFF])          # no inf, NaN = S.1111.111
    assert d[0x80] == 0.0 and math.copysign(1, d[0x80]) == -1


def test_e4m3_decode_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = nm.e4m3_decode(np.arange(256))
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    m = ~np.isnan(ref)
    assert np.array_equal(ref[m], got[m])


def test_e4m3_encode_roundtrip_all_finite_codes():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = nm.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(nm.e4m3_encode(vals), codes)


def test_e4m3_encode_ties_to_even_between_neighbours():
    pos = [c for c in range(0x7F)]
    vals = nm.e4m3_decode(np.array(pos))
    for c in range(len(pos) - 1):
        mid = np.float32((vals[c] + vals[c + 1]) / 2)      # exact in fp32
        want = c if c % 2 == 0 else c + 1                   # even mantissa LSB wins
        assert nm.e4m3_encode(mid) == want, (c, mid)
        assert nm.e4m3_encode(-mid) == (want | 0x80)
        lo = np.nextafter(mid, np.float32(-np.inf), dtype=np.float32)
        hi = np.nextafter(mid, np.float32(np.inf), dtype=np.float32)
        assert nm.e4m3_encode(lo) == c and nm.e4m3_encode(hi) == c + 1


def test_e4m3_encode_saturates_and_nan():
    big = np.array([448.0, 460.0, 464.0, 479.0, 480.0, 1e6, 3e38, np.inf], np.float32)
    assert np.all(nm.e4m3_encode(big) == 0x7E)
    assert np.all(nm.e4m3_encode(-big) == 0xFE)
    assert nm.e4m3_encode(np.float32(np.nan)) == 0x7F


def test_e4m3_encode_matches_torch_cast_in_range():
    g = torch.Generator().manual_seed(2)
    x = (torch.randn(300000, generator=g) * torch.exp(torch.randn(300000, generator=g) * 3)).clamp(-448, 448)
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = nm.e4m3_encode(x.numpy())
    nz = x.numpy() != 0
    assert np.array_equal(ref[nz], got[nz])


# ---------------------------------------------------------------- activation / weight quant

def _bf16(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(torch.bfloat16).to(torch.float64).numpy()


def test_quant_act_amax_maps_to_448_and_error_bound():
    y = _bf16((64, 300), 3)                       # 3 groups, last one 44 wide
    q, s = ov.quant_act(y)
    assert q.shape == y.shape and s.shape == (3, 64) and s.dtype == np.float32
    deq = ov.dequant_act(q, s)
    for g in range(3):
        blk = y[:, g * 128:(g + 1) * 128]
        amax = np.abs(blk).max(1)
        assert np.allclose(s[g], amax / 448.0, rtol=2 ** -23)
        # the largest-magnitude element encodes to +-448 exactly
        idx = np.abs(blk).argmax(1)
        codes = q[np.arange(64), g * 128 + idx]
        assert np.all((codes & 0x7F) == 0x7E)
    # reconstruction: half an E4M3 ulp (2**-4 relative) or half a subnormal step
    err = np.abs(deq - y)
    col_s = np.repeat(s.astype(np.float64), 128, 0)[:300].T
    bound = np.maximum(np.abs(y) * 2.0 ** -4, col_s * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(err <= bound)


def test_quant_act_zero_group_and_power_of_two_invariance():
    y = _bf16((8, 256), 4)
    y[3, :128] = 0.0
    q, s = ov.quant_act(y)
    assert s[0, 3] == 0 and np.all(q[3, :128] == 0)
    for k in (-5, 3, 9):
        q2, s2 = ov.quant_act(y * 2.0 ** k)
        assert np.array_equal(q, q2)
        assert np.array_equal(s2, (s * np.float32(2.0 ** k)).astype(np.float32))


def test_quant_act_zero_padding_changes_nothing():
    """Zero-padding K (e.g. 4304 -> 4352) leaves every code and scale unchanged."""
    y = _bf16((5, 4304), 5)
    q, s = ov.quant_act(y)
    qp, sp = ov.quant_act(np.concatenate([y, np.zeros((5, 48))], 1))
    assert np.array_equal(q, qp[:, :4304]) and np.all(qp[:, 4304:] == 0)
    assert np.array_equal(s, sp)


def test_quant_weight_blocks_are_independent():
    w = _bf16((200, 260), 6, 0.02)
    q, s = ov.quant_weight(w)
    assert s.shape == (2, 3)
    w2 = w.copy()
    w2[150, 10] = 5.0                              # lives in block (1, 0)
    q2, s2 = ov.quant_weight(w2)
    changed = s2 != s
    assert changed[1, 0] and changed.sum() == 1
    same = np.ones_like(q, bool)
    same[128:, :128] = False
    assert np.array_equal(q[same], q2[same])
    # per block, the block amax -> 448 and the block transpose of quant_act agrees
    qt, st = ov.quant_act(w[:128, :128].T.copy())
    assert np.isclose(st.max(), s[0, 0], rtol=0) or st.max() <= s[0, 0]


# ---------------------------------------------------------------- GEMM

def _brute_gemm(qa, sa, qw, sw, bias, res):
    M, K = qa.shape
    N = qw.shape[0]
    out = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            tot = 0.0
            for kb in range(-(-K // 128)):
                part = 0
                for k in range(kb * 128, min(K, kb * 128 + 128)):
                    part += float(nm.e4m3_decode(qa[m, k])) * float(nm.e4m3_decode(qw[n, k]))
                tot += float(sa[kb, m]) * float(sw[n // 128, kb]) * part
            out[m, n] = tot + float(bias[n]) + float(res[m, n])
    return out


def test_gemm_matches_brute_force_loops():
    g = np.random.default_rng(7)
    M, N, K = 3, 130, 260                          # N and K both cross a 128 block with a tail
    qa = g.integers(0, 256, (M, K)).astype(np.uint8)
    qw = g.integers(0, 256, (N, K)).astype(np.uint8)
    qa[(qa & 0x7F) == 0x7F] = 0x10
    qw[(qw & 0x7F) == 0x7F] = 0x22
    sa = g.random((3, M)).astype(np.float32) * 0.01
    sw = g.random((2, 3)).astype(np.float32) * 0.001
    bias = nm.bf16_round(g.standard_normal(N) * 0.1)
    res = nm.bf16_round(g.standard_normal((M, N)))
    got = ov.fp8_block_gemm(qa, sa, qw, sw, bias, res)
    ref = _brute_gemm(qa, sa, qw, sw, bias, res)
    # one bf16 rounding of (nearly) the exact value
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-30)
    assert np.array_equal(got, nm.bf16_round(ref)) or np.mean(got != nm.bf16_round(ref)) < 0.01


def test_gemm_exact_integer_case():
    # codes of small integers, unit scales: the product is an exact integer matrix
    ints = {1: 0x38, 2: 0x40, 3: 0x44, -1: 0xB8, 0: 0x00}
    g = np.random.default_rng(8)
    A = g.choice([1, 2, 3, -1, 0], (4, 256))
    W = g.choice([1, 2, 3, -1, 0], (5, 256))
    qa = np.vectorize(ints.get)(A).astype(np.uint8)
    qw = np.vectorize(ints.get)(W).astype(np.uint8)
    out = ov.fp8_block_gemm(qa, np.ones((2, 4), np.float32), qw, np.ones((1, 2), np.float32))
    # exact integers, then the one bf16 rounding of the output (8 significant bits)
    assert np.array_equal(out, nm.bf16_round((A @ W.T).astype(np.float64)))
    small = np.clip(A, -1, 1), np.clip(W, -1, 1)            # |sum| <= 256: exact in bf16
    out2 = ov.fp8_block_gemm(np.vectorize(ints.get)(small[0]).astype(np.uint8), np.ones((2, 4), np.float32),
                             np.vectorize(ints.get)(small[1]).astype(np.uint8), np.ones((1, 2), np.float32))
    assert np.array_equal(out2, (small[0] @ small[1].T).astype(np.float64))


def test_gemm_operand_orientation():
    """A single nonzero code in A[m, k] and W[n, k] lands at C[m, n] only."""
    qa = np.zeros((4, 128), np.uint8)
    qw = np.zeros((6, 128), np.uint8)
    qa[2, 17] = 0x38
    qw[5, 17] = 0x40
    out = ov.fp8_block_gemm(qa, np.full((1, 4), 3.0, np.float32), qw, np.full((1, 1), 0.5, np.float32))
    want = np.zeros((4, 6))
    want[2, 5] = 3.0 * 0.5 * 2.0
    assert np.array_equal(out, want)


def test_bf16_gemm_matches_brute_force_loops():
    """Every output is the bf16 rounding of an exactly summed dot product + bias + residual
    (bf16 x bf16 products are exact in fp64; the sums are checked with Python's exact fsum)."""
    g = np.random.default_rng(17)
    M, N, K = 3, 10, 37
    a = nm.bf16_round(g.standard_normal((M, K)))
    w = nm.bf16_round(g.standard_normal((N, K)) * 0.1)
    bias = nm.bf16_round(g.standard_normal(N) * 0.1)
    res = nm.bf16_round(g.standard_normal((M, N)))
    got = ov.bf16_gemm(a, w, bias, res)
    for m in range(M):
        for n in range(N):
            exact = math.fsum([float(a[m, k]) * float(w[n, k]) for k in range(K)] + [float(bias[n]), float(res[m, n])])
            assert abs(got[m, n] - exact) <= abs(exact) * 2.0 ** -8 + 1e-30


def test_bf16_gemm_exact_integer_case_and_orientation():
    g = np.random.default_rng(18)
    A = g.integers(-3, 4, (4, 64)).astype(np.float64)
    W = g.integers(-3, 4, (5, 64)).astype(np.float64)
    assert np.array_equal(ov.bf16_gemm(A, W), nm.bf16_round(A @ W.T))   # exact integers, one rounding
    a = np.zeros((4, 16))
    w = np.zeros((6, 16))
    a[2, 9], w[5, 9] = 3.0, 0.5
    out = ov.bf16_gemm(a, w, bias=np.arange(6.0), residual=np.full((4, 6), 2.0))
    want = np.tile(np.arange(6.0) + 2.0, (4, 1))
    want[2, 5] += 1.5
    assert np.array_equal(out, want)


# ---------------------------------------------------------------- position embedding

def test_pos_interp_at_table_resolution_is_the_table():
    g = np.random.default_rng(21)
    table = g.standard_normal((48 * 48, 5))
    assert np.array_equal(ov.pos_embed_interp(table, 48, 48).reshape(-1, 5), table)


def test_pos_interp_reproduces_affine_tables():
    """Bilinear interpolation is exact on a table affine in (row, col) (and on constants)."""
    i, j = np.meshgrid(np.arange(48.0), np.arange(48.0), indexing="ij")
    table = np.stack([3.0 + 0.0 * i, 2.0 * i - 0.5 * j + 1.0, 0.25 * i * 1.0], -1).reshape(-1, 3)
    for h, w in ((16, 16), (36, 27), (46, 136), (1, 7), (5, 1)):
        out = ov.pos_embed_interp(table, h, w)
        r = np.arange(h)[:, None] * (47.0 / (h - 1) if h > 1 else 0.0)
        c = np.arange(w)[None, :] * (47.0 / (w - 1) if w > 1 else 0.0)
        assert np.allclose(out[..., 0], 3.0, atol=1e-12)
        assert np.allclose(out[..., 1], 2.0 * r - 0.5 * c + 1.0, atol=1e-10)
        assert np.allclose(out[..., 2], 0.25 * r + 0 * c, atol=1e-10)


def test_pos_interp_corner_points_and_midpoints():
    """Corners take the table's corners; a grid of 95 puts every other point halfway between
    two table rows, where the value is the mean of the two."""
    g = np.random.default_rng(22)
    table = g.standard_normal((48 * 48, 2))
    T = table.reshape(48, 48, 2)
    out = ov.pos_embed_interp(table, 95, 48)
    assert np.allclose(out[0, 0], T[0, 0]) and np.allclose(out[-1, -1], T[-1, -1])
    assert np.allclose(out[1], 0.5 * (T[0] + T[1]), atol=1e-12)
    assert np.allclose(out[2], T[1], atol=1e-12)


def test_patch_embed_adds_each_patch_its_own_position():
    """With zero pixels and bias, x is the bf16 position embedding of each token's (row, col)
    in token order (2x2-block order for even grids, row-major for odd)."""
    i, j = np.meshgrid(np.arange(48.0), np.arange(48.0), indexing="ij")
    table = np.stack([i, j], -1).reshape(-1, 2)
    grids = [(4, 6), (3, 5)]
    n = sum(h * w for h, w in grids)
    x = ov.patch_embed(np.zeros((n, 8)), np.zeros((2, 8)), np.zeros(2), table, grids)
    pos, _ = ov.packed_positions(grids)
    want = []
    for (h, w), start in ((grids[0], 0), (grids[1], 24)):
        rc = pos[start:start + h * w]
        want.append(np.stack([rc[:, 0] * 47.0 / (h - 1), rc[:, 1] * 47.0 / (w - 1)], -1))
    assert np.array_equal(x, nm.bf16_round(np.concatenate(want)))


# ---------------------------------------------------------------- LayerNorm / GELU

def test_layernorm_moments_and_affine():
    x = _bf16((16, 1152), 9, 3.0) + 5.0
    y = ov.layernorm_f64(x, np.ones(1152), np.zeros(1152))
    assert np.allclose(y.mean(1), 0, atol=1e-12)
    assert np.allclose(y.var(1), 1 - 1e-6 / (x.var(1) + 1e-6), atol=1e-9)
    g = np.linspace(0.5, 1.5, 1152)
    b = np.linspace(-1, 1, 1152)
    assert np.allclose(ov.layernorm_f64(x, g, b), y * g + b, atol=1e-12)
    # brute force on one row
    r = x[3]
    mu = sum(r) / len(r)
    var = sum((v - mu) ** 2 for v in r) / len(r)
    assert abs(y[3, 10] - (r[10] - mu) / math.sqrt(var + 1e-6)) < 1e-12


def test_gelu_identities():
    x = np.linspace(-8, 8, 2001)
    gl = ov.gelu_tanh_f64(x)
    assert ov.gelu_tanh_f64(0.0) == 0.0
    assert np.allclose(gl - ov.gelu_tanh_f64(-x), x, atol=1e-12)       # odd part is x/2 twice
    assert abs(ov.gelu_tanh_f64(1.0) - 0.5 * (1 + math.tanh(math.sqrt(2 / math.pi) * 1.044715))) < 1e-15
    assert np.allclose(ov.gelu_tanh_f64(np.array([30.0, -30.0])), [30.0, 0.0])
    # equals the tanh form where that form is accurate, and stays accurate beyond it
    xm = np.linspace(-4, 4, 801)
    tanh_form = 0.5 * xm * (1 + np.tanh(math.sqrt(2 / math.pi) * (xm + 0.044715 * xm ** 3)))
    assert np.allclose(ov.gelu_tanh_f64(xm), tanh_form, rtol=1e-10, atol=1e-300)   # tanh form loses digits as x -> -4
    x8 = -8.0                                       # 1 + tanh(u) cancels completely here in fp64
    u8 = math.sqrt(2 / math.pi) * (x8 + 0.044715 * x8 ** 3)
    assert abs(ov.gelu_tanh_f64(x8) - x8 * math.exp(2 * u8) / (1 + math.exp(2 * u8))) <= 1e-15 * abs(ov.gelu_tanh_f64(x8))
    # tanh-GELU stays within 1e-3 of the exact erf GELU on [-8, 8]
    erf_gelu = 0.5 * x * (1 + np.array([math.erf(v / math.sqrt(2)) for v in x]))
    assert np.max(np.abs(gl - erf_gelu)) < 1e-3


# ---------------------------------------------------------------- RoPE and patch order

def test_rope_frequencies():
    f = ov.rope_inv_freq(72, 10000.0)
    assert f.shape == (18,)                         # head_dim / 4 frequencies
    assert f[0] == 1.0 and np.isclose(f[1], 10000 ** (-1 / 18)) and np.isclose(f[17], 10000 ** (-34 / 36))


def test_rope_identity_at_origin_and_norm_preserved():
    g = np.random.default_rng(10)
    x = g.standard_normal((5, 2, 72))
    pos = np.array([[0, 0], [3, 7], [40, 1], [0, 135], [45, 135]])
    ang = ov.rope_angles(pos)
    y = ov.rope_rotate(x, ang)
    assert np.allclose(y[0], x[0], atol=0)
    pn = lambda t: t[..., :36] ** 2 + t[..., 36:] ** 2  # noqa: E731
    assert np.allclose(pn(y), pn(x), rtol=1e-12, atol=1e-12)


def test_rope_relative_position_property():
    g = np.random.default_rng(11)
    q = g.standard_normal(72)
    k = g.standard_normal(72)

    def dot(p, pp):
        a = ov.rope_rotate(q[None], ov.rope_angles(np.array([p])))[0]
        b = ov.rope_rotate(k[None], ov.rope_angles(np.array([pp])))[0]
        return a @ b
    assert np.isclose(dot((3, 5), (1, 2)), dot((10, 20), (8, 17)), rtol=1e-10)
    assert not np.isclose(dot((3, 5), (1, 2)), dot((3, 5), (2, 1)), rtol=1e-6)


def test_rope_rotate_half_pairing_brute_force():
    g = np.random.default_rng(12)
    x = g.standard_normal(72)
    pos = (6, 11)
    y = ov.rope_rotate(x[None], ov.rope_angles(np.array([pos])))[0]
    f = [10000 ** (-2 * i / 36) for i in range(18)]
    for j in range(36):
        a = (pos[0] * f[j]) if j < 18 else (pos[1] * f[j - 18])
        assert abs(y[j] - (x[j] * math.cos(a) - x[j + 36] * math.sin(a))) < 1e-12
        assert abs(y[j + 36] - (x[j + 36] * math.cos(a) + x[j] * math.sin(a))) < 1e-12


def test_patch_order_2x2_blocks_and_coverage():
    for h, w in ((16, 16), (46, 136), (54, 18), (2, 4)):
        p = ov.patch_positions(h, w)
        assert len({tuple(r) for r in p}) == h * w
        assert p[:, 0].max() == h - 1 and p[:, 1].max() == w - 1
        quads = p.reshape(-1, 4, 2)
        base = quads[:, 0]
        assert np.all(base % 2 == 0)
        assert np.all(quads - base[:, None] == np.array([[0, 0], [0, 1], [1, 0], [1, 1]]))
    p = ov.patch_positions(36, 27)                  # odd: row-major
    assert np.array_equal(p[28], [1, 1]) and np.array_equal(p[-1], [35, 26])


# ---------------------------------------------------------------- attention

def _brute_attn(qkv, cu, heads, d):
    n = qkv.shape[0]
    t = qkv.reshape(n, 3, heads, d)
    out = np.zeros((n, heads, d))
    for a, b in zip(cu[:-1], cu[1:]):
        for h in range(heads):
            for i in range(a, b):
                s = [sum(t[i, 0, h, e] * t[j, 1, h, e] for e in range(d)) / math.sqrt(d) for j in range(a, b)]
                mx = max(s)
                p = [math.exp(v - mx) for v in s]
                z = sum(p)
                for e in range(d):
                    out[i, h, e] = sum(p[j - a] * t[j, 2, h, e] for j in range(a, b)) / z
    return out.reshape(n, heads * d)


def test_attention_matches_brute_force():
    g = np.random.default_rng(13)
    heads, d = 2, 8
    cu = [0, 5, 6, 13]
    qkv = nm.bf16_round(g.standard_normal((13, 3 * heads * d)) * 2)
    got = ov.attention_varlen(qkv, cu, heads, d)
    ref = _brute_attn(qkv, cu, heads, d)
    assert np.array_equal(got, nm.bf16_round(ref)) or np.max(np.abs(got - ref)) <= np.abs(ref).max() * 2 ** -8


def test_attention_single_key_returns_v_and_segments_independent():
    g = np.random.default_rng(14)
    heads, d = 3, 72
    qkv = nm.bf16_round(g.standard_normal((20, 3 * heads * d)))
    cu = [0, 1, 9, 20]
    out = ov.attention_varlen(qkv, cu, heads, d)
    v0 = qkv[0].reshape(3, heads, d)[2].reshape(-1)
    assert np.array_equal(out[0], v0)
    for a, b in zip(cu[:-1], cu[1:]):
        alone = ov.attention_varlen(qkv[a:b], [0, b - a], heads, d)
        assert np.array_equal(alone, out[a:b])


def test_attention_permutation_equivariance():
    g = np.random.default_rng(15)
    heads, d = 2, 72
    qkv = nm.bf16_round(g.standard_normal((33, 3 * heads * d)))
    perm = g.permutation(33)
    a = ov.attention_varlen(qkv, [0, 33], heads, d)
    b = ov.attention_varlen(qkv[perm], [0, 33], heads, d)
    assert np.allclose(a[perm], b, rtol=2 ** -7, atol=1e-6)


def test_softmax_rows_sum_to_one_via_constant_v():
    g = np.random.default_rng(16)
    heads, d = 2, 72
    qkv = g.standard_normal((40, 3 * heads * d)) * 4
    t = qkv.reshape(40, 3, heads, d)
    t[:, 2] = 1.0                                   # v = 1: output = row sum of softmax
    out = ov.attention_varlen(t.reshape(40, -1), [0, 17, 40], heads, d)
    assert np.all(out == 1.0)


# ---------------------------------------------------------------- merger shape pins

def test_merger_concatenates_four_consecutive_rows():
    x = _bf16((8, 4), 17)
    g = np.ones(16)
    b = np.zeros(16)
    ref = ov.layernorm(np.stack([np.concatenate(x[4 * i:4 * i + 4]) for i in range(2)]), g, b)
    assert np.array_equal(ov.layernorm(x.reshape(2, 16), g, b), ref)
