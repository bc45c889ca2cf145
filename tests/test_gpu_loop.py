"""The decode-time cycle on the GPU, in both redundancy modes: tokens are appended
(rkv_append_kv) until the buffer is full, the step compresses back to the budget
(rkv_compress_step), and so on.  Every compression is checked against the oracle on the cache as it
was just before the step; the whole cycle is also captured in a CUDA graph and
must replay bit for bit like the eager calls."""
import numpy as np
import pytest
import torch

import oracle
from rkv_synth import bf16_bits
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu

L, B, H, G, D = 2, 2, 2, 4, 128
BUDGET, BUFFER, WINDOW = 96, 32, 8
CAP = BUDGET + BUFFER


@pytest.fixture(scope="module")
def rkv(cuda_device):
    from decode_kv_cache_head_b200 import build
    build.build()
    import decode_kv_cache_head_b200 as m
    return m


def _trace(seed, T):
    """New keys / values / queries of T decode steps: AR(1) keys with repeated
    segments, so that near duplicates appear as they do in reasoning traces."""
    g = torch.Generator().manual_seed(seed)
    eps = torch.randn((L, B, H, T, D), generator=g)
    k = torch.empty_like(eps)
    k[..., 0, :] = eps[..., 0, :]
    for t in range(1, T):
        k[..., t, :] = 0.9 * k[..., t - 1, :] + (1 - 0.81) ** 0.5 * eps[..., t, :]
    rng = np.random.default_rng(seed)
    for p in range(40, T - 16, 37):
        n = int(rng.integers(4, 12))
        s = int(rng.integers(0, p - n))
        k[..., p:p + n, :] = k[..., s:s + n, :] + 0.01 * torch.randn((L, B, H, n, D), generator=g)
    v = torch.randn((L, B, H, T, D), generator=g)
    q = torch.randn((L, B, H * G, T, D), generator=g)
    return k.to(torch.bfloat16), v.to(torch.bfloat16), q.to(torch.bfloat16)


@pytest.mark.parametrize("red_mode", [0, 1], ids=["mean", "max"])
def test_append_then_compress_cycles_match_the_oracle(rkv, red_mode):
    dev = torch.device("cuda")
    T = CAP + 5 * BUFFER
    kt, vt, qt = _trace(81, T)
    cfg = rkv.make_config(BUDGET, BUFFER, WINDOW, D, H, H * G, 0.1, redundancy_mode=red_mode)
    K = torch.zeros((L, B, H, CAP, D), dtype=torch.bfloat16, device=dev)
    V = torch.zeros_like(K)
    cur = torch.zeros(B, dtype=torch.int32, device=dev)
    ws = torch.zeros(rkv.rkv_workspace_size(cfg, L, B, CAP), dtype=torch.uint8, device=dev)
    t = 0
    steps = 0
    while t < T:
        n_new = CAP - int(cur[0]) if steps == 0 else BUFFER
        k_new = kt[:, :, :, t:t + n_new].contiguous().to(dev)
        v_new = vt[:, :, :, t:t + n_new].contiguous().to(dev)
        rkv.rkv_append_kv(cfg, K, V, k_new, v_new, cur, ws)
        t += n_new
        assert cur.tolist() == [CAP] * B
        # queries of the window: the last WINDOW decode steps
        Q = qt[:, :, :, t - WINDOW:t].contiguous().to(dev)
        before_k, before_v = K.clone(), V.clone()
        kept = torch.full((L, B, H, CAP), -1, dtype=torch.int32, device=dev)
        rkv.rkv_compress_step(cfg, K, V, Q, cur, ws, kept_out=kept)
        torch.cuda.synchronize()
        assert rkv.rkv_workspace_status(ws) == 0
        assert cur.tolist() == [BUDGET] * B
        kb, qb = bf16_bits(before_k), bf16_bits(Q)
        kh = kept.cpu().numpy()
        for l in range(L):
            for b in range(B):
                for h in range(H):
                    o = oracle.unit(qb[l, b, h * G:(h + 1) * G], kb[l, b, h], CAP, BUDGET, 0.1,
                                    red_mode=red_mode)
                    kp = kh[l, b, h, :BUDGET]
                    gc.check_kept_layout(kp, CAP - WINDOW, CAP, BUDGET)
                    gc.boundary_check(o["Z"], kp[:BUDGET - WINDOW], BUDGET - WINDOW)
                    gc.check_compaction(before_k[l, b, h], K[l, b, h], kp, BUDGET)
                    gc.check_compaction(before_v[l, b, h], V[l, b, h], kp, BUDGET)
        steps += 1
    assert steps == 6


@pytest.mark.parametrize("red_mode", [0, 1], ids=["mean", "max"])
def test_the_cycle_replays_in_a_cuda_graph(rkv, red_mode):
    dev = torch.device("cuda")
    kt, vt, qt = _trace(82, CAP + 4 * BUFFER)
    cfg = rkv.make_config(BUDGET, BUFFER, WINDOW, D, H, H * G, 0.1, redundancy_mode=red_mode)

    def fresh():
        K = torch.zeros((L, B, H, CAP, D), dtype=torch.bfloat16, device=dev)
        V = torch.zeros_like(K)
        K[..., :BUDGET, :] = kt[..., :BUDGET, :].to(dev)
        V[..., :BUDGET, :] = vt[..., :BUDGET, :].to(dev)
        return K, V, torch.full((B,), BUDGET, dtype=torch.int32, device=dev)

    k_new = torch.empty((L, B, H, BUFFER, D), dtype=torch.bfloat16, device=dev)
    v_new = torch.empty_like(k_new)
    Q = torch.empty((L, B, H * G, WINDOW, D), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(rkv.rkv_workspace_size(cfg, L, B, CAP), dtype=torch.uint8, device=dev)

    def feed(i):
        t = BUDGET + i * BUFFER
        k_new.copy_(kt[..., t:t + BUFFER, :])
        v_new.copy_(vt[..., t:t + BUFFER, :])
        Q.copy_(qt[..., t + BUFFER - WINDOW:t + BUFFER, :])

    # eager reference
    Ke, Ve, ce = fresh()
    for i in range(4):
        feed(i)
        rkv.rkv_append_kv(cfg, Ke, Ve, k_new, v_new, ce, ws)
        rkv.rkv_compress_step(cfg, Ke, Ve, Q, ce, ws)
    torch.cuda.synchronize()

    # the same cycle as one captured graph, replayed four times
    Kg, Vg, cg_ = fresh()
    feed(0)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            rkv.rkv_append_kv(cfg, Kg, Vg, k_new, v_new, cg_, ws, stream=s)
            rkv.rkv_compress_step(cfg, Kg, Vg, Q, cg_, ws, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    Kg2, Vg2, cg2 = fresh()      # capture does not run the work: start over
    Kg.copy_(Kg2); Vg.copy_(Vg2); cg_.copy_(cg2)
    for i in range(4):
        feed(i)
        graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(cg_, ce)
    assert torch.equal(Kg.view(torch.int16), Ke.view(torch.int16))
    assert torch.equal(Vg.view(torch.int16), Ve.view(torch.int16))
