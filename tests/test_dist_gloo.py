"""Multi-rank host logic on CPU (gloo, world size 2): the timing and sharding plumbing the
benchmark uses when each GPU runs its own sequences."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from sparse_attention_long_fwd_b200 import dist as nd


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    try:
        w, r, loc = nd.init("gloo", timeout_s=30)
        assert (w, r, loc) == (world, rank, rank)
        nd.barrier(w)
        # each rank measured a different step time; every rank must see the slowest
        mx = nd.max_over_ranks(1.5 + rank, w)
        start, count = nd.shard(64, r, w)
        rate = nd.aggregate_rate(131072, w, mx)
        q.put((rank, mx, start, count, rate))
    finally:
        if torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


def test_two_rank_timing_and_sharding():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [2.5, 2.5]                 # max over ranks
    assert [(r[2], r[3]) for r in res] == [(0, 32), (32, 32)]  # contiguous halves of 64 sequences
    assert all(abs(r[4] - 2 * 131072 / 2.5) < 1e-6 for r in res)


@pytest.mark.parametrize("total,world", [(64, 3), (5, 8), (0, 2), (131072, 8)])
def test_shard_covers_every_unit_once(total, world):
    spans = [nd.shard(total, r, world) for r in range(world)]
    assert sum(c for _, c in spans) == total
    pos = 0
    for s, c in spans:
        assert s == pos
        pos += c
    assert max(c for _, c in spans) - min(c for _, c in spans) <= 1


def test_single_process_defaults():
    assert nd.rank_env() == (1, 0, 0) or "WORLD_SIZE" in os.environ
    assert nd.max_over_ranks(3.0, 1) == 3.0
