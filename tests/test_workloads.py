"""The seeded input recipe: shapes, dtypes, determinism, distinct seeds, and the
distributions the design notes state (x ~ N(0, s^2) per image; weights N(0, 0.02);
biases N(0, 0.01); gamma = 1 + N(0, 0.02))."""
import torch

from quantized_vit_encoder_b200 import workloads as wl


def _std_close(t, std, rel=0.05):
    return abs(t.float().std().item() - std) <= rel * std


def test_workload_table():
    W = wl.WORKLOADS
    assert [W[k].n_tokens for k in ("block_16x16", "block_36x27", "block_46x136", "tower_46x136",
                                    "tower_packed4")] == [256, 972, 6256, 6256, 9164]
    p = W["tower_packed4"]
    offsets = [0]
    for h, w in p.grids:
        offsets.append(offsets[-1] + h * w)
    assert offsets == [0, 972, 7228, 8140, 9164]
    assert all(h % 2 == 0 and w % 2 == 0 for h, w in p.grids)
    assert p.input_scales == (0.1, 1.0, 10.0, 1.0) and W["tower_46x136"].input_scales == (1.0,)
    assert W["tower_46x136"].n_blocks == wl.N_BLOCKS == 27 and W["tower_46x136"].mergers


def test_seeds_are_distinct_within_and_across_workloads():
    seeds = []
    for W in wl.WORKLOADS.values():
        seeds.append(W.seed_base)
        seeds += [wl.block_seed(W, b) for b in range(W.n_blocks)]
        seeds += [wl.merger_seed(W, t) for t in range(4)] if W.mergers else []
    assert len(seeds) == len(set(seeds))


def test_inputs_are_deterministic_and_follow_the_recipe():
    W = wl.WORKLOADS["tower_packed4"]
    x = wl.make_input(W)
    assert x.dtype == torch.bfloat16 and x.shape == (9164, wl.HIDDEN)
    assert torch.equal(x, wl.make_input(W))
    a = 0
    for (h, w), s in zip(W.grids, W.input_scales):
        assert _std_close(x[a:a + h * w], s, 0.02)
        a += h * w
    assert not torch.equal(wl.random_bf16((64, 64), 1), wl.random_bf16((64, 64), 2))


def test_weights_follow_the_recipe():
    p = wl.block_params(7)
    assert torch.equal(p["qkv_w"], wl.block_params(7)["qkv_w"])
    assert all(v.dtype == torch.bfloat16 for v in p.values())
    for k in ("qkv_w", "proj_w", "fc1_w", "fc2_w"):
        assert _std_close(p[k], wl.W_STD) and abs(p[k].float().mean().item()) < 1e-3
    for k in ("qkv_b", "proj_b", "fc1_b", "fc2_b", "norm1_b", "norm2_b"):
        assert _std_close(p[k], wl.B_STD, 0.15)
    for k in ("norm1_w", "norm2_w"):
        assert abs(p[k].float().mean().item() - 1.0) < 3e-3 and _std_close(p[k] - 1, wl.GAMMA_STD, 0.15)
    m = wl.merger_params(8)
    assert m["fc1_w"].shape == (4608, 4608) and m["fc2_w"].shape == (2048, 4608)
    assert _std_close(m["fc1_w"], wl.W_STD) and _std_close(m["norm_w"] - 1, wl.GAMMA_STD, 0.15)
    q = wl.patch_params(9)
    assert q["w"].shape == (1152, 1536) and q["pos"].shape == (48 * 48, 1152)
