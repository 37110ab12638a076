"""Host logic of the multi-GPU bench (N independent replicas): rank discovery, barrier and the
max-over-ranks reduction of the timed duration, run as 2 gloo ranks on the CPU."""

import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench

    w, r, lr = bench.dist_env()
    assert (w, r, lr) == (world, rank, rank)
    dist = bench.init_dist(world, "gloo")
    bench.barrier(world)
    # each rank reports a different duration; everyone must see the maximum
    got = bench.max_over_ranks(1.5 + rank, world)
    out[rank] = got
    bench.barrier(world)
    dist.destroy_process_group()


def test_two_rank_max_and_barrier():
    torch = pytest.importorskip("torch")
    import torch.multiprocessing as mp

    world = 2
    port = _free_port()
    manager = mp.Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert dict(out) == {0: 2.5, 1: 2.5}


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.25, 1) == 3.25
    bench.barrier(1)  # no-op
