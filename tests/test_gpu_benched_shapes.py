"""Parity at the launch shapes the benchmark times, on every unit of the
Llama3-8B-shaped step (32 layers x 8 KV heads, N = 1152, 8 queries per head
window, G = 4):

* MAX redundancy (the similarity kernel at 256 units) for lambda = 0, 0.1, 1,
  with the undecided fraction of each printed;
* paged caches with 16-row pages, MEAN against the oracle and MAX bit-identical
  to the contiguous MAX step;
* shared selection with the KV heads split over two emulated tensor-parallel
  ranks (the partial scores summed, as the all-reduce does).
"""
import numpy as np
import pytest
import torch

import oracle
from rkv_synth import WORKLOADS, bf16_bits, make_inputs
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu

W = WORKLOADS["llama3_8b_step"]


@pytest.fixture(scope="module")
def rkv(cuda_device):
    from decode_kv_cache_head_b200 import build
    build.build()
    import decode_kv_cache_head_b200 as m
    return m


@pytest.fixture(scope="module")
def inputs():
    x = make_inputs(W)
    units = [(l, 0, h) for l in range(W.n_layers) for h in range(W.n_kv_heads)]
    return x, units


def _cfg(rkv, lam, red_mode, heads=None):
    H = heads or W.n_kv_heads
    G = W.n_q_heads // W.n_kv_heads
    return rkv.make_config(W.budget_of(0), W.buffer, W.window, 128, H, H * G, lam,
                           redundancy_mode=red_mode)


def _step(rkv, cfg, x):
    dev = torch.device("cuda")
    K, V, Q = x["K"].to(dev).clone(), x["V"].to(dev).clone(), x["Q"].to(dev)
    cur = x["cur_len"].to(dev).clone()
    L, B, H, cap, _ = K.shape
    ws = torch.zeros(rkv.rkv_workspace_size(cfg, L, B, cap), dtype=torch.uint8, device=dev)
    kept = torch.full((L, B, H, cap), -1, dtype=torch.int32, device=dev)
    scores = torch.zeros((L, B, H, 4, cap), dtype=torch.float32, device=dev)
    rkv.rkv_compress_step(cfg, K, V, Q, cur, ws, kept_out=kept, scores_out=scores)
    torch.cuda.synchronize()
    assert rkv.rkv_workspace_status(ws) == 0
    assert cur.tolist() == [W.budget_of(0)]
    return K, V, kept.cpu().numpy(), scores.cpu().numpy()


def _verify(x, units, K, V, kept, sc, orc):
    N, bud = int(x["cur_len"][0]), W.budget_of(0)
    M = N - W.window
    und = []
    for i, (l, b, h) in enumerate(units):
        gc.check_scores("M*I", sc[l, b, h, 0, :M], orc["I"][i, :M], scale=M)
        gc.check_scores("r", sc[l, b, h, 1, :M], orc["r"][i, :M])
        gc.check_scores("M*R", sc[l, b, h, 2, :M], orc["R"][i, :M], scale=M)
        kp = kept[l, b, h, :bud]
        gc.check_kept_layout(kp, M, N, bud)
        und.append(gc.boundary_check(orc["Z"][i, :M], kp[:bud - W.window], bud - W.window))
        gc.check_compaction(x["K"][l, b, h], K[l, b, h], kp, bud)
        gc.check_compaction(x["V"][l, b, h], V[l, b, h], kp, bud)
    return float(np.mean(und))


@pytest.mark.parametrize("lam", [0.0, 0.1, 1.0])
def test_max_redundancy_every_unit(rkv, inputs, lam):
    x, units = inputs
    K, V, kept, sc = _step(rkv, _cfg(rkv, lam, 1), x)
    orc = gc.oracle_for_units(x["K"], x["Q"], units, lambda b: int(x["cur_len"][b]),
                              W.budget_of, lambda b: lam, 4, red_mode=oracle.RED_MAX)
    und = _verify(x, units, K, V, kept, sc, orc)
    print(f"MAX redundancy, lambda {lam}: undecided fraction {und:.4f}")


def _paged(rkv, cfg, x, P, perm_seed=7):
    dev = torch.device("cuda")
    L, B, H, cap, D = x["K"].shape
    mb = cap // P
    pages = B * mb + 5                                   # spare pages, never touched
    perm = torch.randperm(pages, generator=torch.Generator().manual_seed(perm_seed))[:B * mb]
    bt = perm.to(torch.int32).view(B, mb).to(dev)
    pk = torch.zeros((L, pages, H, P, D), dtype=torch.bfloat16, device=dev)
    pv = torch.zeros_like(pk)
    idx = bt.view(-1).long()
    pk[:, idx] = x["K"].to(dev).view(L, B, H, mb, P, D).permute(0, 1, 3, 2, 4, 5).reshape(L, B * mb, H, P, D)
    pv[:, idx] = x["V"].to(dev).view(L, B, H, mb, P, D).permute(0, 1, 3, 2, 4, 5).reshape(L, B * mb, H, P, D)
    ws = torch.zeros(rkv.rkv_workspace_size(cfg, L, B, cap), dtype=torch.uint8, device=dev)
    freed = torch.full((B, mb), -1, dtype=torch.int32, device=dev)
    n_freed = torch.zeros((B,), dtype=torch.int32, device=dev)
    kept = torch.full((L, B, H, cap), -1, dtype=torch.int32, device=dev)
    scores = torch.zeros((L, B, H, 4, cap), dtype=torch.float32, device=dev)
    cur = x["cur_len"].to(dev).clone()
    rkv.rkv_compress_step_paged(cfg, pk, pv, x["Q"].to(dev), cur, ws, bt, P, freed, n_freed,
                                kept_out=kept, scores_out=scores)
    torch.cuda.synchronize()
    assert rkv.rkv_workspace_status(ws) == 0
    # back to the contiguous layout
    K = pk[:, idx].view(L, B, mb, H, P, D).permute(0, 1, 3, 2, 4, 5).reshape(L, B, H, cap, D)
    V = pv[:, idx].view(L, B, mb, H, P, D).permute(0, 1, 3, 2, 4, 5).reshape(L, B, H, cap, D)
    return K, V, kept.cpu().numpy(), scores.cpu().numpy(), freed.cpu().numpy(), n_freed.cpu().numpy(), bt.cpu().numpy()


def test_paged_16_row_pages_every_unit(rkv, inputs):
    x, units = inputs
    P = 16
    K, V, kept, sc, freed, n_freed, bt = _paged(rkv, _cfg(rkv, 0.1, 0), x, P)
    orc = gc.oracle_for_units(x["K"], x["Q"], units, lambda b: int(x["cur_len"][b]),
                              W.budget_of, lambda b: 0.1, 4)
    und = _verify(x, units, K, V, kept, sc, orc)
    print(f"paged P = 16: undecided fraction {und:.4f}")
    N, bud = int(x["cur_len"][0]), W.budget_of(0)
    first, last = -(-bud // P), -(-N // P)
    assert n_freed[0] == last - first
    assert list(freed[0, :last - first]) == list(bt[0, first:last])


def test_paged_max_redundancy_matches_the_contiguous_step(rkv, inputs):
    x, _ = inputs
    cfg = _cfg(rkv, 0.1, 1)
    Kc, Vc, kc, sc = _step(rkv, cfg, x)
    Kp, Vp, kp, sp, _, _, _ = _paged(rkv, cfg, x, 16, perm_seed=11)
    np.testing.assert_array_equal(kp, kc)
    np.testing.assert_array_equal(sp, sc)           # r from the similarity kernel, bit for bit
    bud = W.budget_of(0)
    assert torch.equal(Kp[..., :bud, :].view(torch.int16).cpu(), Kc[..., :bud, :].view(torch.int16).cpu())
    assert torch.equal(Vp[..., :bud, :].view(torch.int16).cpu(), Vc[..., :bud, :].view(torch.int16).cpu())


@pytest.mark.parametrize("red_mode", [0, 1], ids=["mean", "max"])
def test_shared_selection_two_ranks_every_layer(rkv, inputs, red_mode):
    x, _ = inputs
    dev = torch.device("cuda")
    L, B, H, cap, _ = x["K"].shape
    G = 4
    parts = []
    for h0, h1 in ((0, 4), (4, 8)):
        K = x["K"][:, :, h0:h1].contiguous().to(dev)
        V = x["V"][:, :, h0:h1].contiguous().to(dev)
        Q = x["Q"][:, :, h0 * G:h1 * G].contiguous().to(dev)
        cur = x["cur_len"].to(dev).clone()
        cfg = _cfg(rkv, 0.1, red_mode, heads=4)
        ws = torch.zeros(rkv.rkv_workspace_size_shared(cfg, L, B, cap), dtype=torch.uint8,
                         device=dev)
        z = torch.empty((L, B, cap), dtype=torch.float32, device=dev)
        rkv.rkv_score_shared(cfg, K, Q, cur, z, ws)
        parts.append(dict(K=K, V=V, cur=cur, cfg=cfg, ws=ws, z=z))
    total = parts[0]["z"] + parts[1]["z"]
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
    assert torch.equal(kepts[0], kepts[1])
    kept = kepts[0].cpu().numpy()
    zs = total.cpu().numpy()
    Kall = torch.cat([parts[0]["K"], parts[1]["K"]], dim=2).cpu()
    Vall = torch.cat([parts[0]["V"], parts[1]["V"]], dim=2).cpu()
    kb, qb = bf16_bits(x["K"]), bf16_bits(x["Q"])
    N, bud = int(x["cur_len"][0]), W.budget_of(0)
    M = N - W.window
    und = []
    for l in range(L):
        q = np.stack([qb[l, 0, h * G:(h + 1) * G] for h in range(H)])
        k = np.stack([kb[l, 0, h] for h in range(H)])
        o = oracle.shared_units(q, k, N, bud, 0.1, red_mode=red_mode, n_threads=gc.n_threads())
        gc.check_scores("M*Zsum/H", zs[l, 0, :M] / H, o["Zsum"] / H, scale=M)
        kp = kept[l, 0, :bud]
        gc.check_kept_layout(kp, M, N, bud)
        und.append(gc.boundary_check(o["Zsum"] / H, kp[:bud - W.window], bud - W.window))
        for h in range(H):
            gc.check_compaction(x["K"][l, 0, h], Kall[l, 0, h], kp, bud)
            gc.check_compaction(x["V"][l, 0, h], Vall[l, 0, h], kp, bud)
    print(f"shared selection ({'max' if red_mode else 'mean'}): undecided fraction "
          f"{np.mean(und):.4f}")
