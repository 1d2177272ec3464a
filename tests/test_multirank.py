"""Host logic of the multi-GPU benchmark on CPU with two gloo ranks: the batch is sharded across
ranks with no data-path collective, and the timing is the max over ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    lo, hi = bench.shard_range(16, world, rank)
    t = bench.max_over_ranks(1.5 + rank, device="cpu")
    dist.barrier()
    q.put((rank, lo, hi, t))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharding_and_max_over_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # shards tile the batch exactly once
    covered = []
    for _, lo, hi, _ in res:
        covered.extend(range(lo, hi))
    assert covered == list(range(16))
    # every rank sees the slowest rank's time
    assert all(t == 1.5 + (world - 1) for *_, t in res)


def test_shard_range_uneven():
    assert [bench.shard_range(10, 3, r) for r in range(3)] == [(0, 4), (4, 7), (7, 10)]
    assert bench.max_over_ranks(2.5) == 2.5
