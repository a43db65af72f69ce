"""Writes tests/golden/drift_bounds.json: how far the oracle's own composite outputs
move when two of its rounding points are perturbed (oracle/perturb.py).  Calls only
oracle/ and the seeded input generator.

    python tests/golden/make_drift_bounds.py [case ...]

The GPU tests allow a composite output (block, merger, tower taps) to differ from
the oracle by at most DRIFT_MARGIN times these figures.
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from oracle import perturb  # noqa: E402
from oracle import vit as ov  # noqa: E402
from quantized_vit_encoder_b200 import workloads as wl  # noqa: E402

OUT = os.path.join(HERE, "drift_bounds.json")


def f64(t):
    return t.float().double().numpy()


def stats(a, b):
    return {"rel_l2": float(np.linalg.norm(a - b) / np.linalg.norm(b)), "max_abs": float(np.abs(a - b).max())}


def block_case(name):
    W = wl.WORKLOADS[name]
    x = f64(wl.make_input(W))
    q = ov.quantize_block_weights({k: f64(v) for k, v in wl.block_params(wl.block_seed(W, 0)).items()})
    pos, cu = ov.packed_positions(W.grids)
    ref = ov.block_forward(x, q, cu, pos)
    with perturb.perturbed():
        alt = ov.block_forward(x, q, cu, pos)
    return stats(alt, ref)


def merger_case(n):
    x = f64(wl.random_bf16((n, 1152), 700 + n, 2.0))
    m = ov.quantize_merger_weights({k: f64(v) for k, v in wl.merger_params(4242).items()})
    ref = ov.merger_forward(x, m)
    with perturb.perturbed():
        alt = ov.merger_forward(x, m)
    return stats(alt, ref)


def tower_case(grids, scales, seed_base):
    W = wl.Workload("tower_case", tuple(grids), wl.N_BLOCKS, True, scales=tuple(scales), seed_base=seed_base)
    x = f64(wl.make_input(W))
    blocks = [ov.quantize_block_weights({k: f64(v) for k, v in wl.block_params(wl.block_seed(W, b)).items()})
              for b in range(wl.N_BLOCKS)]
    mergers = [ov.quantize_merger_weights({k: f64(v) for k, v in wl.merger_params(wl.merger_seed(W, t)).items()})
               for t in range(4)]
    ref = ov.tower_forward(x, blocks, mergers, W.grids)
    with perturb.perturbed():
        alt = ov.tower_forward(x, blocks, mergers, W.grids)
    return [stats(a, r) for a, r in zip(alt, ref)]


def block_bf16_case(name):
    W = wl.WORKLOADS[name]
    x = f64(wl.make_input(W))
    w = {k: f64(v) for k, v in wl.block_params(wl.block_seed(W, 0)).items()}
    pos, cu = ov.packed_positions(W.grids)
    ref = ov.block_forward_bf16(x, w, cu, pos)
    with perturb.perturbed():
        alt = ov.block_forward_bf16(x, w, cu, pos)
    return stats(alt, ref)


def merger_bf16_case(n):
    x = f64(wl.random_bf16((n, 1152), 700 + n, 2.0))
    m = {k: f64(v) for k, v in wl.merger_params(4242).items()}
    ref = ov.merger_forward_bf16(x, m)
    with perturb.perturbed():
        alt = ov.merger_forward_bf16(x, m)
    return stats(alt, ref)


def tower_mixed_case(grids, scales, seed_base):
    W = wl.Workload("tower_case", tuple(grids), wl.N_BLOCKS, True, scales=tuple(scales), seed_base=seed_base)
    x = f64(wl.make_input(W))
    blocks = []
    for b in range(wl.N_BLOCKS):
        p = {k: f64(v) for k, v in wl.block_params(wl.block_seed(W, b)).items()}
        blocks.append(p if b < 3 else ov.quantize_block_weights(p))
    mergers = [{k: f64(v) for k, v in wl.merger_params(wl.merger_seed(W, t)).items()} for t in range(4)]
    ref = ov.tower_forward(x, blocks, mergers, W.grids)
    with perturb.perturbed():
        alt = ov.tower_forward(x, blocks, mergers, W.grids)
    return [stats(a, r) for a, r in zip(alt, ref)]


CASES = {
    "block_bf16_16x16": lambda: block_bf16_case("block_16x16"),
    "block_bf16_36x27": lambda: block_bf16_case("block_36x27"),
    "merger_bf16_972": lambda: merger_bf16_case(972),
    "tower_mixed_small": lambda: tower_mixed_case([(16, 16), (8, 12)], [1.0, 3.0], 5200),
    "block_16x16": lambda: block_case("block_16x16"),
    "block_36x27": lambda: block_case("block_36x27"),
    "block_46x136": lambda: block_case("block_46x136"),
    "merger_4": lambda: merger_case(4),
    "merger_972": lambda: merger_case(972),
    "merger_6256": lambda: merger_case(6256),
    "tower_small": lambda: tower_case([(16, 16), (8, 12)], [1.0, 3.0], 5000),
    "tower_smoke_16x16": lambda: tower_case([(16, 16)], [1.0], 7000),
}


def main(names):
    data = json.load(open(OUT)) if os.path.exists(OUT) else {}
    for name in names or CASES:
        data[name] = CASES[name]()
        print(name, data[name], flush=True)
        json.dump(data, open(OUT, "w"), indent=1, sort_keys=True)


if __name__ == "__main__":
    main(sys.argv[1:])
