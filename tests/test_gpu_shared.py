"""GPU parity of the shared (cross-head / cross-rank) selection against the
oracle: rkv_score_shared, the sum over ranks, rkv_select_compact_shared.  Two
tensor-parallel ranks are emulated on one GPU by two calls on the two halves of
the KV heads whose partial scores are added (what the all-reduce computes); no
kernel waits on another."""
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


def _cfg(rkv, w, lam, red_mode=0, heads=None, budget=None):
    H = heads or w.n_kv_heads
    G = w.n_q_heads // w.n_kv_heads
    return rkv.make_config(budget or w.budget_of(0), w.buffer, w.window, 128, H, H * G, lam,
                           redundancy_mode=red_mode)


def _oracle_shared(x, l, b, N, budget, lam, G, red_mode=0):
    kb, qb = bf16_bits(x["K"]), bf16_bits(x["Q"])
    H = kb.shape[2]
    q = np.stack([qb[l, b, h * G:(h + 1) * G] for h in range(H)])
    k = np.stack([kb[l, b, h] for h in range(H)])
    return oracle.shared_units(q, k, N, budget, lam, red_mode=red_mode, n_threads=gc.n_threads())


def _check(w, x, K, V, kept, z_sum, budgets, lam, red_mode=0, due=lambda b: True):
    G = w.n_q_heads // w.n_kv_heads
    H = w.n_kv_heads
    for l in range(w.n_layers):
        for b in range(w.batch):
            if not due(b):
                continue
            N, bud = int(x["cur_len"][b]), budgets[b]
            M = N - w.window
            o = _oracle_shared(x, l, b, N, bud, lam, G, red_mode)
            # scores: the head sum, in the unit-mean scale (M * Zsum / H)
            gc.check_scores("M*Zsum/H", z_sum[l, b, :M] / H, o["Zsum"] / H, scale=M)
            assert np.all(z_sum[l, b, M:] == 0)
            kp = kept[l, b, :bud]
            gc.check_kept_layout(kp, M, N, bud)
            gc.boundary_check(o["Zsum"] / H, kp[:bud - w.window], bud - w.window)
            for h in range(H):
                gc.check_compaction(x["K"][l, b, h], K[l, b, h], kp, bud)
                gc.check_compaction(x["V"][l, b, h], V[l, b, h], kp, bud)


def _run(rkv, cfg, K, V, Q, cur, z, ws, budgets=None, kept=None):
    rkv.rkv_score_shared(cfg, K, Q, cur, z, ws, budgets=budgets)
    rkv.rkv_select_compact_shared(cfg, K, V, cur, z, ws, budgets=budgets, kept_out=kept)


@pytest.mark.parametrize("red_mode,lam", [(0, 0.1), (0, 1.0), (1, 0.1)])
def test_one_rank(rkv, red_mode, lam):
    w = Workload("sh", 2, 2, 4, 16, 128, (512, 300), buffer=100, seed=91)
    x = make_inputs(w)
    dev = torch.device("cuda")
    K, V, Q = x["K"].to(dev).clone(), x["V"].to(dev).clone(), x["Q"].to(dev)
    cur = x["cur_len"].to(dev).clone()
    L, B, H, cap, _ = K.shape
    cfg = _cfg(rkv, w, lam, red_mode)
    budgets_h = [512, 300]
    budgets = torch.tensor(budgets_h, dtype=torch.int32, device=dev)
    ws = torch.zeros(rkv.rkv_workspace_size_shared(cfg, L, B, cap), dtype=torch.uint8, device=dev)
    z = torch.full((L, B, cap), float("nan"), dtype=torch.float32, device=dev)
    kept = torch.full((L, B, cap), -1, dtype=torch.int32, device=dev)
    _run(rkv, cfg, K, V, Q, cur, z, ws, budgets, kept)
    torch.cuda.synchronize()
    assert rkv.rkv_workspace_status(ws) == 0
    assert cur.tolist() == budgets_h
    _check(w, x, K, V, kept.cpu().numpy(), z.cpu().numpy(), budgets_h, lam, red_mode)


def test_two_ranks_evict_the_identical_set(rkv):
    """Heads 0-3 on one rank, 4-7 on the other: after the partial scores are summed
    both ranks keep the same rows, and those are the one-rank result's up to ties."""
    w = Workload("tp", 3, 2, 8, 32, 128, (1024,), seed=92)
    x = make_inputs(w)
    dev = torch.device("cuda")
    L, B, H, cap, _ = x["K"].shape
    G = 4
    halves = [(0, 4), (4, 8)]
    parts = []
    for h0, h1 in halves:
        K = x["K"][:, :, h0:h1].contiguous().to(dev)
        V = x["V"][:, :, h0:h1].contiguous().to(dev)
        Q = x["Q"][:, :, h0 * G:h1 * G].contiguous().to(dev)
        cur = x["cur_len"].to(dev).clone()
        cfg = _cfg(rkv, w, 0.1, heads=4)
        ws = torch.zeros(rkv.rkv_workspace_size_shared(cfg, L, B, cap), dtype=torch.uint8,
                         device=dev)
        z = torch.empty((L, B, cap), dtype=torch.float32, device=dev)
        rkv.rkv_score_shared(cfg, K, Q, cur, z, ws)
        parts.append(dict(K=K, V=V, cur=cur, cfg=cfg, ws=ws, z=z))
    total = parts[0]["z"] + parts[1]["z"]          # the all-reduce (sum) of two ranks
    kepts = []
    for p in parts:
        p["z"].copy_(total)
        kept = torch.full((L, B, cap), -1, dtype=torch.int32, device=dev)
        rkv.rkv_select_compact_shared(p["cfg"], p["K"], p["V"], p["cur"], p["z"], p["ws"],
                                      kept_out=kept)
        kepts.append(kept)
    torch.cuda.synchronize()
    for p in parts:
        assert rkv.rkv_workspace_status(p["ws"]) == 0
        assert p["cur"].tolist() == [1024, 1024]
    assert torch.equal(kepts[0], kepts[1])
    Kall = torch.cat([parts[0]["K"], parts[1]["K"]], dim=2).cpu()
    Vall = torch.cat([parts[0]["V"], parts[1]["V"]], dim=2).cpu()
    _check(w, x, Kall, Vall, kepts[0].cpu().numpy(), total.cpu().numpy(), [1024, 1024], 0.1)


def test_not_due_and_disabled(rkv):
    w = Workload("nd", 1, 3, 2, 8, 128, (256, 256, 256), seed=93)
    x = make_inputs(w)
    dev = torch.device("cuda")
    K, V, Q = x["K"].to(dev).clone(), x["V"].to(dev).clone(), x["Q"].to(dev)
    cur = x["cur_len"].to(dev).clone()
    cur[1] -= 5                                     # not due
    budgets = torch.tensor([256, 256, 0], dtype=torch.int32, device=dev)   # 2: disabled
    L, B, H, cap, _ = K.shape
    cfg = _cfg(rkv, w, 0.1)
    ws = torch.zeros(rkv.rkv_workspace_size_shared(cfg, L, B, cap), dtype=torch.uint8, device=dev)
    z = torch.full((L, B, cap), 7.0, dtype=torch.float32, device=dev)
    kept = torch.full((L, B, cap), -1, dtype=torch.int32, device=dev)
    before = cur.tolist()
    _run(rkv, cfg, K, V, Q, cur, z, ws, budgets, kept)
    torch.cuda.synchronize()
    assert cur.tolist() == [256, before[1], before[2]]
    zs = z.cpu()
    assert torch.all(zs[:, 1:] == 0)                # defined zeros where nothing is due
    for b in (1, 2):
        assert torch.equal(K[:, b].cpu(), x["K"][:, b]) and torch.equal(V[:, b].cpu(), x["V"][:, b])
    x2 = dict(x, cur_len=x["cur_len"])
    _check(w, x2, K.cpu(), V.cpu(), kept.cpu().numpy(), z.cpu().numpy(), [256, 256, 256], 0.1,
           due=lambda b: b == 0)
