"""The multi-rank host logic on CPU: two gloo ranks on 127.0.0.1."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from decode_kv_cache_head_b200 import dist as rdist


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world_size, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world_size)
    try:
        ws, r = rdist.world()
        start, stop = rdist.shard_range(5, ws, r)
        # each rank reports a different "time"; everyone must see the max
        m = rdist.max_over_ranks([1.0 + r, 10.0 - r], torch.device("cpu"))
        rdist.barrier(torch.device("cpu"))
        out[r] = (ws, r, start, stop, m, rdist.rank_seed(2, r))
    finally:
        dist.destroy_process_group()


def test_two_rank_sharding_and_max_timing():
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    r0, r1 = out[0], out[1]
    assert (r0[0], r0[1]) == (2, 0) and (r1[0], r1[1]) == (2, 1)
    assert (r0[2], r0[3], r1[2], r1[3]) == (0, 3, 3, 5)   # 5 sequences: 3 + 2, contiguous
    assert r0[4] == r1[4] == [2.0, 10.0]
    assert r0[5] != r1[5]


def test_single_process_defaults():
    assert rdist.world() == (1, 0)
    assert rdist.shard_range(7, 1, 0) == (0, 7)
    assert rdist.max_over_ranks([3.0], torch.device("cpu")) == [3.0]
    for n in range(0, 20):
        for ws in range(1, 5):
            parts = [rdist.shard_range(n, ws, r) for r in range(ws)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            assert all(parts[i][1] == parts[i + 1][0] for i in range(ws - 1))
