"""The N > 1 bench path on CPU: two gloo ranks, each with its own independent workload (weak
scaling, no collective on the data path), and the max-over-ranks reduction of step times."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from block_sparse_attention_pbsa_b200 import inputs as I


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
