"""Two gloo ranks on CPU: the benchmark's sequence sharding and max-over-ranks timing."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, B, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from kv_cache_attention_fdllm_b200.shard import max_over_ranks, rank_sequences
        mine = rank_sequences(B, rank)
        allseq = [None] * world
        dist.all_gather_object(allseq, mine)
        t = max_over_ranks(1.5 + rank)
        q.put((rank, allseq, t))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_sequences_and_reduce_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, 3, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, allseq, t in res:
        assert allseq[0] == [0, 1, 2] and allseq[1] == [3, 4, 5]   # disjoint, covers 0..5
        assert t == 2.5                                            # max over ranks


def test_max_over_ranks_without_group():
    from kv_cache_attention_fdllm_b200.shard import max_over_ranks
    assert max_over_ranks(3.25) == 3.25
