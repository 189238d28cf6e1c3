"""The N > 1 paths on CPU with gloo ranks: the bench's weak scaling (each rank its own
independent workload, no collective on the data path) and the max-over-ranks reduction of
step times; and the head partition of one layer across ranks (each rank its heads' share of
the layer, no exchange inside the step), checked against the whole layer."""
import dataclasses
import os
import socket

import numpy as np
import pytest

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from block_sparse_attention_pbsa_b200 import inputs as I
from block_sparse_attention_pbsa_b200 import shard


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.rank_workload(I.DECODE_5S, rank)
        # a stand-in per-rank step time; the reduction must return the slowest rank's value
        mine = 0.25 + rank * 0.5
        out[rank] = (w.seed, bench.max_over_ranks(mine, torch.device("cpu"), world))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling_and_max():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    seeds = [res[r][0] for r in range(world)]
    assert len(set(seeds)) == world            # independent problems per rank
    assert all(res[r][1] == 0.75 for r in range(world))


def test_head_ranges_partition_every_layer():
    for heads in (1, 5, 12, 24, 30):
        for world in range(1, min(heads, 9) + 1):
            ranges = [shard.head_range(heads, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == heads
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))          # contiguous, disjoint
            sizes = [h1 - h0 for h0, h1 in ranges]
            assert max(sizes) - min(sizes) <= 1 and sorted(sizes, reverse=True) == sizes
    assert [shard.head_range(12, 8, r) for r in range(8)][:5] == [(0, 2), (2, 4), (4, 6), (6, 8), (8, 9)]
    with pytest.raises(ValueError):
        shard.head_range(4, 5, 0)


# a small layer for the oracle: 6 heads, 16x32-token frames (8 blocks each), 8 history frames
SMALL = dataclasses.replace(I.DECODE_5S, heads=6, head_dim=16, frame_h=16, frame_w=32, hist_frames=8,
                            chunk_frames=2, capacity=16, window_frames=3, topk=5, seed=11)


def _plan(w, q, k, kc):
    from oracle import pbsa_oracle as O
    gd = {"frame_h": w.frame_h, "frame_w": w.frame_w, "tile_h": w.tile_h, "tile_w": w.tile_w, "scale": w.scale}
    f = lambda t: t.double().numpy()  # noqa: E731
    p = O.single_step_plan(f(q), f(k), gd, w.hist_frames, w.chunk_frames, w.capacity, w.window_frames,
                           w.topk, w.gamma, k_chunk=f(kc))
    return {key: p[key] for key in ("P", "sel", "P2")}


def _shard_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = SMALL
        q, k, _ = I.single_step(w)
        kc = I.tokens(w, w.chunk_frames, I.stream_seed(w.seed, 4))
        mine = [shard.head_slice(t, w.heads, world, rank) for t in (q, k, kc)]
        wl = dataclasses.replace(w, heads=mine[0].shape[1])
        got = [None] * world
        dist.all_gather_object(got, (shard.head_range(w.heads, world, rank), _plan(wl, *mine)))
        if rank == 0:
            out["parts"] = got
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_head_partition_equals_the_whole_layer(world):
    """Each gloo rank runs the oracle's chunk decode plan (bootstrap update, local selections,
    post-chunk update) on its heads only; gathered over the ranks, the per-head results equal
    the whole layer's (the path needs no exchange between heads)."""
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_shard_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        parts = out["parts"]
    w = SMALL
    q, k, _ = I.single_step(w)
    kc = I.tokens(w, w.chunk_frames, I.stream_seed(w.seed, 4))
    whole = _plan(w, q, k, kc)
    seen = []
    for (h0, h1), plan in parts:
        seen += list(range(h0, h1))
        for key in ("P", "sel", "P2"):
            assert plan[key] == whole[key][h0:h1], (key, h0, h1)
    assert seen == list(range(w.heads))
