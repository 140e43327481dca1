"""Multi-process host logic of the benchmark on CPU (gloo, world size 2): the
mixer shards by sequence with no exchange step, so ranks share only the
barrier and the max over ranks of the timed region."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank  # this rank's timed region
        bench.barrier(world)
        worst = bench.max_over_ranks(ms, world, device="cpu")
        shard = bench.shard_sequences([5000, 100, 3000, 2000, 70, 64], world, rank)
        q.put((rank, worst, shard))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_max_and_shard_disjointly():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]
    shards = [set(r[2]) for r in res]
    assert shards[0].isdisjoint(shards[1]) and shards[0] | shards[1] == set(range(6))


def test_shard_sequences_balances_tokens():
    lengths = [32768, 1024, 20000, 5000, 15000, 8000, 1024, 30000]
    parts = [bench.shard_sequences(lengths, 4, r) for r in range(4)]
    assert sorted(i for p in parts for i in p) == list(range(8))
    loads = [sum(lengths[i] for i in p) for p in parts]
    assert max(loads) <= sum(lengths) / 4 + max(lengths)
