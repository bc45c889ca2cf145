"""GPU parity of the per-head entry points (one sequence and layer, all KV
heads) against the oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from rkv_synth import Workload, bf16_bits, make_inputs
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rkv(cuda_device):
    from decode_kv_cache_head_b200 import build
    build.build()
    import decode_kv_cache_head_b200 as m
    return m


def _case(n_kv, n_q, budget, buffer, window, seed, dup=0.3):
    w = Workload("t", 1, 1, n_kv, n_q, 128, (budget,), buffer=buffer, window=window,
                 dup_frac=(dup,), seed=seed)
    x = make_inputs(w)
    return w, x


# (n_kv, n_q, budget, buffer, window): several tiles per CTA, ragged tails, G=5, tiny N
SHAPES = [
    (8, 32, 1024, 128, 8),     # N = 1152, the Llama3-8B step shape
    (2, 10, 2048, 128, 8),     # N = 2176, G = 5
    (2, 8, 870, 130, 8),       # N = 1000, not a multiple of 16
    (1, 4, 24, 16, 8),         # N = 40
    (2, 2, 300, 77, 1),        # G = 1, w = 1
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("pool", [0, 1])
def test_importance_and_inv_norm(rkv, shape, pool):
    n_kv, n_q, budget, buffer, window = shape
    w, x = _case(n_kv, n_q, budget, buffer, window, seed=31 + budget)
    N = budget + buffer
    M = N - window
    G = n_q // n_kv
    cfg = rkv.make_config(budget, buffer, window, 128, n_kv, n_q, 0.1, gqa_pool=pool)
    dev = torch.device("cuda")
    q = x["Q"][0, 0].to(dev)
    k = x["K"][0, 0].to(dev)
    I = torch.empty((n_kv, M), dtype=torch.float32, device=dev)
    inv = torch.empty((n_kv, N), dtype=torch.float32, device=dev)
    ws = torch.zeros(rkv.rkv_workspace_size(cfg, 1, 1, w.cap), dtype=torch.uint8, device=dev)
    rkv.rkv_score_importance(cfg, q, k, N, I, inv, ws)
    assert rkv.rkv_workspace_status(ws) == 0
    qb, kb = bf16_bits(x["Q"][0, 0]), bf16_bits(x["K"][0, 0])
    for h in range(n_kv):
        want = oracle.importance(qb[h * G:(h + 1) * G], kb[h], N, pool)
        gc.check_scores(f"M*I head {h}", I[h].cpu().numpy(), want, scale=M)
        np.testing.assert_allclose(inv[h].cpu().numpy(), oracle.inv_norm(kb[h], N), rtol=2e-6)


@pytest.mark.parametrize("shape", SHAPES)
def test_redundancy_mean(rkv, shape):
    n_kv, n_q, budget, buffer, window = shape
    w, x = _case(n_kv, n_q, budget, buffer, window, seed=41 + budget)
    N = budget + buffer
    M = N - window
    cfg = rkv.make_config(budget, buffer, window, 128, n_kv, n_q, 0.1)
    dev = torch.device("cuda")
    k = x["K"][0, 0].to(dev)
    r = torch.empty((n_kv, M), dtype=torch.float32, device=dev)
    R = torch.empty((n_kv, M), dtype=torch.float32, device=dev)
    ws = torch.zeros(rkv.rkv_workspace_size(cfg, 1, 1, w.cap), dtype=torch.uint8, device=dev)
    rkv.rkv_score_redundancy(cfg, k, N, r, R, ws)
    kb = bf16_bits(x["K"][0, 0])
    for h in range(n_kv):
        rr = oracle.redundancy(kb[h], N, window, oracle.RED_MEAN)
        gc.check_scores(f"r head {h}", r[h].cpu().numpy(), rr)
        gc.check_scores(f"M*R head {h}", R[h].cpu().numpy(), oracle.softmax(rr), scale=M)


@pytest.mark.parametrize("lam", [0.0, 0.1, 1.0])
@pytest.mark.parametrize("shape", SHAPES[:4])
def test_select_matches_oracle_on_the_same_fp32_scores(rkv, shape, lam):
    """Scores fed in, so the select is isolated from scoring error: the kept
    set must equal the oracle's selection on the identical fp32 Z."""
    n_kv, n_q, budget, buffer, window = shape
    w, x = _case(n_kv, n_q, budget, buffer, window, seed=51 + budget)
    N = budget + buffer
    M = N - window
    G = n_q // n_kv
    qb, kb = bf16_bits(x["Q"][0, 0]), bf16_bits(x["K"][0, 0])
    I32 = np.stack([oracle.importance(qb[h * G:(h + 1) * G], kb[h], N) for h in range(n_kv)]
                   ).astype(np.float32)
    R32 = np.stack([oracle.softmax(oracle.redundancy(kb[h], N, window)) for h in range(n_kv)]
                   ).astype(np.float32)
    cfg = rkv.make_config(budget, buffer, window, 128, n_kv, n_q, lam)
    dev = torch.device("cuda")
    kept = torch.full((n_kv, budget), -1, dtype=torch.int32, device=dev)
    Z = torch.empty((n_kv, M), dtype=torch.float32, device=dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    rkv.rkv_select_topk(cfg, torch.from_numpy(I32).to(dev), torch.from_numpy(R32).to(dev), N,
                        kept, Z, ws)
    lam32 = np.float32(lam)
    Zh = np.float32(lam32 * I32) - np.float32(np.float32(np.float32(1.0) - lam32) * R32)
    np.testing.assert_array_equal(Z.cpu().numpy(), Zh)
    for h in range(n_kv):
        want = oracle.select(Zh[h].astype(np.float64), N, budget)
        np.testing.assert_array_equal(kept[h].cpu().numpy(), want)


def test_select_ties_and_empty_candidate_set(rkv):
    dev = torch.device("cuda")
    N, window = 300, 8
    M = N - window
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    I = torch.full((1, M), 1.0 / M, device=dev)
    R = torch.full((1, M), 1.0 / M, device=dev)
    for budget in (window, 100, N - 1, N):
        cfg = rkv.make_config(budget, 128, window, 128, 1, 4, 0.1)
        kept = torch.full((1, budget), -1, dtype=torch.int32, device=dev)
        rkv.rkv_select_topk(cfg, I, R, N, kept, None, ws)
        kk = budget - window
        assert kept[0].tolist() == list(range(kk)) + list(range(M, N))


@pytest.mark.parametrize("in_place", [False, True])
@pytest.mark.parametrize("budget,N", [(1024, 1152), (2048, 2176), (37, 64), (3000, 3100)])
def test_compaction_bit_exact(rkv, in_place, budget, N):
    dev = torch.device("cuda")
    n_kv, cap = 3, N + 5
    g = torch.Generator(device="cpu").manual_seed(budget)
    K = torch.randn((n_kv, cap, 128), generator=g).to(torch.bfloat16).to(dev)
    V = torch.randn((n_kv, cap, 128), generator=g).to(torch.bfloat16).to(dev)
    kept = torch.stack([torch.sort(torch.randperm(N, generator=g)[:budget]).values
                        for _ in range(n_kv)]).to(torch.int32).to(dev)
    want_k = torch.stack([K[h, kept[h].long()] for h in range(n_kv)])
    want_v = torch.stack([V[h, kept[h].long()] for h in range(n_kv)])
    cfg = rkv.make_config(budget, 128, 8, 128, n_kv, n_kv * 4, 0.1)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    if in_place:
        rkv.rkv_compact_kv(cfg, K, V, kept, K, V, N, ws)
        got_k, got_v = K[:, :budget], V[:, :budget]
    else:
        Kd, Vd = torch.zeros_like(K), torch.zeros_like(V)
        rkv.rkv_compact_kv(cfg, K, V, kept, Kd, Vd, N, ws)
        got_k, got_v = Kd[:, :budget], Vd[:, :budget]
    assert rkv.rkv_workspace_status(ws) == 0
    assert torch.equal(got_k.view(torch.int16), want_k.view(torch.int16))
    assert torch.equal(got_v.view(torch.int16), want_v.view(torch.int16))


def test_compaction_flags_out_of_range_index(rkv):
    """An index past n_tokens is skipped and reported through the workspace."""
    dev = torch.device("cuda")
    K = torch.zeros((1, 64, 128), dtype=torch.bfloat16, device=dev)
    V = torch.zeros_like(K)
    kept = torch.arange(32, dtype=torch.int32, device=dev)[None].clone()
    kept[0, 5] = 1000
    cfg = rkv.make_config(32, 16, 8, 128, 1, 4, 0.1)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    Kd, Vd = torch.zeros_like(K), torch.zeros_like(V)
    rkv.rkv_compact_kv(cfg, K, V, kept, Kd, Vd, 48, ws)
    assert rkv.rkv_workspace_status(ws) == -9


@pytest.mark.parametrize("shape", SHAPES)
def test_redundancy_max_on_the_tensor_cores(rkv, shape):
    """MAX mode: r_i = max over the other keys of the cosine similarity (tcgen05 Gram)."""
    n_kv, n_q, budget, buffer, window = shape
    w, x = _case(n_kv, n_q, budget, buffer, window, seed=71 + budget)
    N = budget + buffer
    M = N - window
    cfg = rkv.make_config(budget, buffer, window, 128, n_kv, n_q, 0.1,
                          redundancy_mode=rkv.RKV_RED_MAX)
    dev = torch.device("cuda")
    k = x["K"][0, 0].to(dev)
    r = torch.empty((n_kv, M), dtype=torch.float32, device=dev)
    R = torch.empty((n_kv, M), dtype=torch.float32, device=dev)
    ws = torch.zeros(rkv.rkv_workspace_size(cfg, 1, 1, w.cap), dtype=torch.uint8, device=dev)
    rkv.rkv_score_redundancy(cfg, k, N, r, R, ws)
    assert rkv.rkv_workspace_status(ws) == 0
    kb = bf16_bits(x["K"][0, 0])
    for h in range(n_kv):
        rr = oracle.redundancy(kb[h], N, window, oracle.RED_MAX)
        gc.check_scores(f"r head {h}", r[h].cpu().numpy(), rr)
        gc.check_scores(f"M*R head {h}", R[h].cpu().numpy(), oracle.softmax(rr), scale=M)


def test_redundancy_max_exact_copies_score_one(rkv):
    dev = torch.device("cuda")
    N, window = 300, 8
    g = torch.Generator(device="cpu").manual_seed(5)
    k = torch.randn((1, N, 128), generator=g).to(torch.bfloat16)
    k[0, 200] = k[0, 17]
    k[0, 250] = k[0, 17] * 4          # same direction, four times longer
    cfg = rkv.make_config(200, 100, window, 128, 1, 4, 0.1, redundancy_mode=rkv.RKV_RED_MAX)
    r = torch.empty((1, N - window), dtype=torch.float32, device=dev)
    ws = torch.zeros(rkv.rkv_workspace_size(cfg, 1, 1, N), dtype=torch.uint8, device=dev)
    rkv.rkv_score_redundancy(cfg, k.to(dev), N, r, None, ws)
    rr = r[0].cpu()
    for i in (17, 200, 250):
        assert abs(float(rr[i]) - 1.0) < 1e-5
    others = torch.ones(N - window, dtype=torch.bool)
    others[[17, 200, 250]] = False
    assert float(rr[others].max()) < 0.5
