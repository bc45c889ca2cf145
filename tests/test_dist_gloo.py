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


def _tp_worker(rank, world_size, port, out):
    """Tensor parallelism over two gloo ranks: each rank scores its own KV heads
    (the oracle stands in for the GPU scoring here), the partial eviction scores
    are summed by the library's all-reduce helper, and each rank selects."""
    import numpy as np

    import oracle
    from rkv_synth import bf16_bits

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world_size)
    try:
        g = torch.Generator().manual_seed(5)
        H, G, w, N, budget = 8, 4, 8, 300, 180
        k = bf16_bits(torch.randn((H, N, 128), generator=g).to(torch.bfloat16))
        q = bf16_bits(torch.randn((H, G, w, 128), generator=g).to(torch.bfloat16))
        h0, h1 = rdist.head_range(H, world_size, rank)
        o = oracle.units(q[h0:h1], k[h0:h1], N, budget, 0.1)
        z = torch.from_numpy(o["Z"][:, :N - w].sum(axis=0).astype(np.float32))
        rdist.allreduce_eviction_scores(z)
        _, kept = oracle.shared_select(z.double().numpy()[None], N, budget)
        out[rank] = (h0, h1, kept.tolist())
    finally:
        dist.destroy_process_group()


def test_tensor_parallel_ranks_evict_the_identical_set():
    import numpy as np

    import oracle
    from rkv_synth import bf16_bits

    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_tp_worker, args=(2, port, out), nprocs=2, join=True)
    (a0, a1, ka), (b0, b1, kb) = out[0], out[1]
    assert (a0, a1, b0, b1) == (0, 4, 4, 8)
    assert ka == kb
    # the same set as one process holding all eight heads
    g = torch.Generator().manual_seed(5)
    k = bf16_bits(torch.randn((8, 300, 128), generator=g).to(torch.bfloat16))
    q = bf16_bits(torch.randn((8, 4, 8, 128), generator=g).to(torch.bfloat16))
    full = oracle.shared_units(q, k, 300, 180, 0.1)
    assert ka == full["kept_shared"].tolist()


def test_head_range():
    assert rdist.head_range(8, 2, 1) == (4, 8)
    assert rdist.head_range(8, 1, 0) == (0, 8)
    with pytest.raises(ValueError):
        rdist.head_range(8, 3, 0)
    z = torch.ones(4)
    assert rdist.allreduce_eviction_scores(z) is z and torch.all(z == 1)
