"""Host-side logic of bench.py that needs no GPU: the max-over-ranks reduction of timings
(world size 2, gloo backend, CPU), the tile pair counts and the blended-roofline FLOP split."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from workloads import CONFIGS


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 5.0 - rank, 3.0 * (rank + 1)]
        out[rank] = bench.reduce_max(mine, "cpu", dist)
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        ps = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in ps:
            p.start()
        for p in ps:
            p.join(timeout=120)
            assert p.exitcode == 0
        assert out[0] == out[1] == [11.0, 5.0, 6.0]


def test_reduce_max_single_process_is_identity():
    assert bench.reduce_max([1.5, 2.5], "cpu", None) == [1.5, 2.5]


@pytest.mark.parametrize("name", ["tiny", "gqa4k", "gemma_local16k"])
def test_tile_pairs_sum_to_visible_pairs(name):
    w = CONFIGS[name]
    assert int(bench.tile_pairs(w).sum()) == w.pairs()


def test_blended_flops_split():
    w = CONFIGS["gqa4k"]
    pairs = bench.tile_pairs(w)
    live = (pairs > 0).astype(np.uint8)
    rmap = np.broadcast_to(live, (w.B, w.H) + live.shape).copy()  # all 8-bit
    F8, F16, F, frac = bench.blended_flops(w, rmap)
    assert F == 4 * w.D * w.pairs() * w.B * w.H
    assert F8 == F16 == F // 2 and frac == 0.0
    rmap[rmap == 1] = 2  # all 16-bit
    F8, F16, F, frac = bench.blended_flops(w, rmap)
    assert F8 == 0 and F16 == F and frac == 1.0


def test_blended_flops_recomputed_tiles_count_both_passes():
    # a tile recomputed by the look-ahead rule (route 3) was scored in 8 bits first: its QK^T
    # counts at both precisions, P.V once
    w = CONFIGS["adaptive8k"].replace(B=1, H=2, Hkv=1, Lq=1024, Lk=1024)
    pairs = bench.tile_pairs(w)
    live = (pairs > 0).astype(np.uint8)
    rmap = np.broadcast_to(live * 3, (w.B, w.H) + live.shape).copy()
    F8, F16, F, frac = bench.blended_flops(w, rmap)
    assert F == 4 * w.D * w.pairs() * w.B * w.H
    assert F8 == F // 2 and F16 == F and frac == 1.0


def test_traffic_record_format():
    # per-workload DRAM traffic of the attention launch (ncu), used only while the kernel
    # sources hash to the recorded value
    import json
    with open(bench.TRAFFIC_FILE) as f:
        tr = json.load(f)
    assert len(tr["kernel_hash"]) == 16
    for name, rec in tr["records"].items():
        assert name in CONFIGS
        assert rec["traffic_bytes_per_launch"] == rec["dram_bytes_read"] + rec["dram_bytes_write"]
