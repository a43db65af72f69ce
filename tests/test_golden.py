"""Pins against numbers printed on the pages (tests/golden/*.txt, each file cites its source)."""
import os

import numpy as np

from oracle import vit as ov
from quantized_vit_encoder_b200 import workloads as wl

HERE = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(HERE, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def test_merger_reduces_patches_four_to_one():
    """Every printed (patches, vision tokens) pair satisfies vision = patches / 4 (2x2 merge)."""
    for patches, llm, text in _rows("patch_token_counts.txt"):
        assert int(patches) % 4 == 0
        assert int(patches) // 4 == int(llm) - int(text)


def test_oracle_merger_output_rows_match_printed_counts():
    """The oracle's merger turns a 6256-patch image (46x136) into 1564 rows, and 972 patches
    (54x18) into 243, as printed."""
    for (h, w), want in (((46, 136), 1564), ((54, 18), 243)):
        pos = ov.patch_positions(h, w)
        assert pos.shape[0] // 4 == want


def test_dims_match_the_pages():
    d = {r[0]: r[1:] for r in _rows("vit_dims.txt")}
    assert int(d["hidden_size"][0]) == wl.HIDDEN
    assert int(d["num_heads"][0]) == wl.HEADS and int(d["head_dim"][0]) == wl.HEAD_DIM
    assert int(d["intermediate_size"][0]) == wl.MLP
    assert int(d["out_hidden_size"][0]) == wl.OUT_HIDDEN
    assert int(d["num_blocks"][0]) == wl.N_BLOCKS
    assert tuple(int(v) for v in d["deepstack_indexes"]) + (int(d["final_merger_after"][0]),) == wl.TAP_AFTER
    assert int(d["rope_inv_freq_len"][0]) == ov.rope_inv_freq(wl.HEAD_DIM).shape[0]
    assert wl.MERGE_IN == int(d["spatial_merge_size"][0]) ** 2 * wl.HIDDEN
    assert np.prod([3, 2, 16, 16]) == int(d["patch_dim"][0])
