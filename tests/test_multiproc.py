"""bench.py's multi-rank host logic on CPU (gloo, world size 2): max-over-ranks timing,
barriers, env parsing, and the reference arm running on rank 0 only."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, l = bench.dist_env()
        assert (w, r, l) == (world, rank, rank)
        bench.barrier(world)
        got = bench.max_over_ranks(1.5 + rank, world, torch.device("cpu"))
        # the reference arm returns nothing on ranks other than 0 (they exit without work)
        class A:
            steps, warmup = 1, 0
        ref = bench.run_reference(A, None) if rank != 0 else "skipped"
        out[rank] = (got, ref)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_barrier():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 2.5
    assert out[1][1] is None
