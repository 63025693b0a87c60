"""The exchange behind the sharded capacity, on CPU with two gloo ranks: every
rank gets all shards' per-expert counts in rank order."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from mixture_experts_layer_54_b200.ops import gather_shard_counts
        counts = torch.arange(5, dtype=torch.int32) * (rank + 1) + 10 * rank
        table = gather_shard_counts(counts)
        q.put((rank, table.tolist()))
    finally:
        dist.destroy_process_group()


def test_gather_shard_counts_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = [[0, 1, 2, 3, 4], [10, 12, 14, 16, 18]]
    assert got[0] == want and got[1] == want
