"""Multi-rank plumbing of the benchmark, on CPU with the gloo backend (world size 2).

The mixer shards over independent sequences, so the only cross-rank operations are the barrier and
the max-over-ranks of the step time; these run here exactly as under NCCL, on CPU tensors.
"""
from __future__ import annotations

import os
import socket

import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, init_method=f"tcp://127.0.0.1:{port}",
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        step_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        out[rank] = bench.reduce_max(step_ms, device="cpu")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_gloo():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        assert dict(out) == {0: 15.0, 1: 15.0}


def test_single_rank_reduce_is_identity():
    assert bench.reduce_max(3.5, device="cpu") == 3.5


def test_rank_shards_are_independent():
    seeds = {bench.shard_seed(1002, r) for r in range(8)}
    assert len(seeds) == 8
