"""Host-side multi-rank logic on CPU (gloo, world size 2): image sharding,
max-over-ranks timing, and that per-rank shards reproduce the packed result
(checked with the oracle on small images)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from quantized_vit_encoder_b200 import replicas


def test_shard_images_covers_all_and_balances():
    grids = [(54, 18), (46, 136), (24, 38), (32, 32)]
    sh = replicas.shard_images(grids, 2)
    assert sorted(i for s in sh for i in s) == list(range(4))
    assert all(s == sorted(s) for s in sh)
    assert sh[0] and sh[1]
    assert replicas.shard_images(grids, 1) == [[0, 1, 2, 3]]
    assert sum(len(s) for s in replicas.shard_images(grids, 8)) == 4
    assert replicas.token_ranges(grids)[-1] == (8140, 9164)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    from oracle import vit as ov
    from quantized_vit_encoder_b200 import workloads as wl
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        grids = [(4, 6), (2, 2), (6, 4)]
        heads, d = 2, 8
        n = sum(h * w for h, w in grids)
        qkv = wl.random_bf16((n, 3 * heads * d), 11).float().double().numpy()
        mine = replicas.shard_images(grids, world)[rank]
        rng = replicas.token_ranges(grids)
        outs = {}
        for i in mine:
            a, b = rng[i]
            outs[i] = ov.attention_varlen(qkv[a:b], [0, b - a], heads, d)
        got = [None] * world
        dist.all_gather_object(got, outs)
        t = replicas.max_over_ranks(float(rank + 1))
        if rank == 0:
            merged = {k: v for o in got for k, v in o.items()}
            full = ov.attention_varlen(qkv, [r[0] for r in rng] + [n], heads, d)
            same = all(np.array_equal(merged[i], full[rng[i][0]:rng[i][1]]) for i in range(len(grids)))
            q.put((same, t, sorted(merged)))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_shards_reproduce_packed_result():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    same, t, keys = q.get(timeout=100)
    for p in procs:
        p.join(timeout=30)
    assert same and t == 2.0 and keys == [0, 1, 2]
