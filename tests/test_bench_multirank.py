"""Host-side logic of bench.py's multi-GPU mode (one process per GPU, each an
independent replica): max-over-ranks timing and the weak-scaling aggregate,
run as world_size-2 gloo process groups on the CPU."""
from __future__ import annotations

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, l = bench.dist_setup()
        assert (w, r, l) == (world, rank, rank)
        # each rank "timed" a different duration; everyone must see the slowest
        ms = bench.max_over_ranks(1.5 + rank)
        val = bench.weak_scaling_value(w, 1e9, ms * 1e-3)
        out[rank] = (ms, val)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_gloo_world2():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 2.5
    assert res[0][1] == res[1][1] == pytest.approx(2 * 1e9 / 2.5e-3)


def test_single_process_is_identity():
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.weak_scaling_value(1, 10.0, 2.0) == 5.0
