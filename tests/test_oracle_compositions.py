"""Pins of the oracle's compositions (block, tower) against closed forms and invariants.

The stage functions are pinned one by one elsewhere; these tests tie the way the
oracle wires them together to facts that hold for the method itself:

* a block whose four linear weights are zero reduces to its two residual adds,
  x2 = bf16(bf16(x + b_proj) + b_fc2) (attention then averages identical v rows,
  which must give the v bias back exactly);
* with such blocks the tower state after block b follows that recursion, so the
  mergers must see the states after blocks 8, 16, 24 and 27 (1-indexed);
* a block over packed images equals the block over each image alone, bit for bit
  (every stage is row-wise except attention, which is per segment);
* the 2x2 merger (FP8 and bf16) normalises the four concatenated rows as one 4608
  row (constant rows give the closed-form values, not the zeros a per-row
  LayerNorm would), maps rows 4i..4i+3 to output row i and nothing else, and ends
  in fc2 with no residual (zero fc2 weights leave exactly its bias).
"""
import numpy as np
import pytest
import torch

from oracle import numerics as nm
from oracle import vit as ov
from quantized_vit_encoder_b200 import workloads as wl

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _f64(t):
    return t.float().double().numpy() if isinstance(t, torch.Tensor) else np.asarray(t, np.float64)


def _zero_linear_block(seed):
    """Block weights with zero linears and the seeded LayerNorm vectors and biases."""
    p = {k: _f64(v) for k, v in wl.block_params(seed).items()}
    for name in ("qkv", "proj", "fc1", "fc2"):
        p[name + "_w"] = np.zeros_like(p[name + "_w"])
    return ov.quantize_block_weights(p)


def test_zero_weight_quantisation_is_all_zero():
    q, s = ov.quant_weight(np.zeros((256, 384)))
    assert not q.any() and not s.any()


@pytest.mark.parametrize("grids", [[(4, 4)], [(3, 5)], [(2, 2), (4, 6)]])
def test_block_with_zero_linears_is_its_residual_adds(grids):
    w = _zero_linear_block(11)
    pos, cu = ov.packed_positions(grids)
    n = pos.shape[0]
    x = _f64(wl.random_bf16((n, 1152), 12, 1.0))
    x2, st = ov.block_forward(x, w, cu, pos, keep=True)
    # the qkv projection is its bias on every row, so attention returns the v bias
    v_b = w["qkv_b"][2304:]
    assert np.array_equal(st["attn"], np.broadcast_to(v_b, (n, 1152)))
    x1 = nm.bf16_round(x + w["proj_b"])
    assert np.array_equal(st["x1"], x1)
    assert np.array_equal(x2, nm.bf16_round(x1 + w["fc2_b"]))


def test_tower_taps_follow_blocks_8_16_24_27(monkeypatch):
    blocks = [_zero_linear_block(100 + b) for b in range(wl.N_BLOCKS)]
    mergers = [ov.quantize_merger_weights({k: _f64(v) for k, v in wl.merger_params(200 + t).items()})
               for t in range(4)]
    grids = [(2, 2)]
    x = _f64(wl.random_bf16((4, 1152), 13, 1.0))
    states = [x]
    for w in blocks:
        x1 = nm.bf16_round(states[-1] + w["proj_b"])
        states.append(nm.bf16_round(x1 + w["fc2_b"]))
    seen = []
    real = ov.merger_forward

    def spy(h, m, eps=1e-6, keep=False):
        seen.append(np.array(h))
        return real(h, m, eps, keep)

    monkeypatch.setattr(ov, "merger_forward", spy)
    taps = ov.tower_forward(x, blocks, mergers, grids)
    assert len(taps) == 4 and len(seen) == 4
    for h, b in zip(seen, (8, 16, 24, 27)):
        assert np.array_equal(h, states[b]), f"merger input is not the state after block {b}"
    for tap, h, m in zip(taps, seen, mergers):
        assert np.array_equal(tap, real(h, m))


def test_block_over_packed_images_equals_each_image_alone():
    w = ov.quantize_block_weights({k: _f64(v) for k, v in wl.block_params(21).items()})
    grids = [(4, 2), (3, 3), (2, 6)]
    pos, cu = ov.packed_positions(grids)
    x = _f64(wl.random_bf16((pos.shape[0], 1152), 22, 1.0))
    packed = ov.block_forward(x, w, cu, pos)
    for i, g in enumerate(grids):
        a, b = int(cu[i]), int(cu[i + 1])
        p1, c1 = ov.packed_positions([g])
        alone = ov.block_forward(x[a:b], w, c1, p1)
        assert np.array_equal(packed[a:b], alone)


def test_bf16_block_with_zero_linears_is_its_residual_adds():
    """The bf16 block of the mixed tower has the same residual wiring as the FP8 block."""
    p = {k: _f64(v) for k, v in wl.block_params(41).items()}
    for name in ("qkv", "proj", "fc1", "fc2"):
        p[name + "_w"] = np.zeros_like(p[name + "_w"])
    pos, cu = ov.packed_positions([(4, 4), (2, 6)])
    n = pos.shape[0]
    x = _f64(wl.random_bf16((n, 1152), 42, 1.0))
    x2 = ov.block_forward_bf16(x, p, cu, pos)
    x1 = nm.bf16_round(x + p["proj_b"])
    assert np.array_equal(x2, nm.bf16_round(x1 + p["fc2_b"]))


def test_mixed_tower_runs_bf16_then_fp8_blocks(monkeypatch):
    """tower_forward dispatches each block on its weights: bf16 weights (no FP8 codes) run
    the bf16 block, quantised weights the FP8 block, in the given order."""
    calls = []
    monkeypatch.setattr(ov, "block_forward", lambda h, w, cu, pos, eps=1e-6: calls.append("fp8") or h)
    monkeypatch.setattr(ov, "block_forward_bf16", lambda h, w, cu, pos, eps=1e-6: calls.append("bf16") or h)
    monkeypatch.setattr(ov, "merger_forward", lambda h, m, eps=1e-6, keep=False: h[: h.shape[0] // 4])
    monkeypatch.setattr(ov, "merger_forward_bf16", lambda h, m, eps=1e-6, keep=False: h[: h.shape[0] // 4])
    bf16_w, fp8_w = {"qkv_w": None}, {"qkv_q": None}
    blocks = [bf16_w] * 3 + [fp8_w] * 24
    mergers = [{"fc1_w": None}] * 4
    ov.tower_forward(np.zeros((4, 1152)), blocks, mergers, [(2, 2)])
    assert calls == ["bf16"] * 3 + ["fp8"] * 24


# ---------------------------------------------------------------- the 2x2 merger

def _merger_weights(seed, fp8=True, **override):
    p = {k: _f64(v) for k, v in wl.merger_params(seed).items()}
    p.update(override)
    return ov.quantize_merger_weights(p) if fp8 else p


def _merger(fp8):
    return ov.merger_forward if fp8 else ov.merger_forward_bf16


def _bf16_of(v):
    """bf16 rounding by torch's cast (independent of the oracle's own rounding)."""
    return torch.tensor(v, dtype=torch.float64).to(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("fp8", [True, False], ids=["fp8", "bf16"])
def test_merger_layernorm_spans_the_four_concatenated_rows(fp8):
    """Four constant rows c_j make one 4608 row whose LayerNorm (gamma 1, beta 0) is
    (c_j - mean) / sqrt(var + eps) on features [1152 j, 1152 (j + 1)): nonzero, where a
    LayerNorm over each 1152 row alone would give zeros, and in the row order."""
    w = _merger_weights(61, fp8, norm_w=np.ones(4608), norm_b=np.zeros(4608))
    groups = [(-3.0, -1.0, 1.0, 3.0), (2.0, 2.0, 2.0, 6.0)]
    x = np.repeat(np.array(groups).reshape(8, 1), 1152, axis=1)
    _, st = _merger(fp8)(x, w, keep=True)
    for g, c in enumerate(groups):
        c = np.array(c)
        v = _bf16_of((c - c.mean()) / np.sqrt(((c - c.mean()) ** 2).mean() + 1e-6))
        if not fp8:
            assert np.array_equal(st["h1"][g], np.repeat(v, 1152))
            continue
        # each 128-column block lies inside one source row, so it is constant: codes +-448
        # and scale fl32(|v_j| / 448)
        blocks = np.repeat(v, 9)
        want_s = (np.abs(blocks).astype(np.float32) / np.float32(448.0)).astype(np.float32)
        assert np.array_equal(st["s1"][:, g], want_s)
        want_q = np.repeat(np.where(blocks > 0, 0x7E, 0xFE), 128).astype(np.uint8)
        assert np.array_equal(st["q1"][g], want_q)


@pytest.mark.parametrize("fp8", [True, False], ids=["fp8", "bf16"])
def test_merger_output_row_depends_on_its_four_rows_only(fp8):
    """Output row i is a function of input rows 4i..4i+3: permuting the groups permutes
    the output rows bit for bit, and changing one input row changes one output row."""
    w = _merger_weights(62, fp8)
    x = _f64(wl.random_bf16((16, 1152), 63, 1.0))
    run = _merger(fp8)
    out = run(x, w)
    perm = [2, 0, 3, 1]
    xp = np.concatenate([x[4 * g:4 * g + 4] for g in perm])
    assert np.array_equal(run(xp, w), out[perm])
    x2 = x.copy()
    x2[5] = _f64(wl.random_bf16((1, 1152), 64, 1.0))[0]
    out2 = run(x2, w)
    changed = [i for i in range(4) if not np.array_equal(out2[i], out[i])]
    assert changed == [1]


@pytest.mark.parametrize("fp8", [True, False], ids=["fp8", "bf16"])
def test_merger_with_zero_fc2_is_its_output_bias(fp8):
    """fc2 is the last step and has no residual: zero fc2 weights leave b_fc2 on every row."""
    w = _merger_weights(65, fp8, fc2_w=np.zeros((2048, 4608)))
    x = _f64(wl.random_bf16((8, 1152), 66, 1.0))
    out = _merger(fp8)(x, w)
    assert np.array_equal(out, np.broadcast_to(w["fc2_b"], (2, 2048)))
