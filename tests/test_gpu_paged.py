"""The step on paged caches (rkv_compress_step_paged): rows scattered over a
page pool through a block table give exactly the contiguous step's result,
match the oracle, and the pages each compressed sequence no longer needs are
handed back."""
import numpy as np
import pytest
import torch

from oracle import rkv_oracle_np as onp
from rkv_synth import Workload, make_inputs
from tests.test_gpu_step import all_units, run_step, verify

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rkv(cuda_device):
    from decode_kv_cache_head_b200 import build
    build.build()
    import decode_kv_cache_head_b200 as m
    return m


def _to_pages(x, P, spare, seed):
    """Scatter the contiguous caches [L, B, H, cap, D] into pools [L, pages, H, P, D]
    with a random page assignment; returns the pools and the block table."""
    K, V = x["K"], x["V"]
    L, B, H, cap, D = K.shape
    assert cap % P == 0
    mb = cap // P
    pages = B * mb + spare
    perm = np.random.default_rng(seed).permutation(pages)
    bt = perm[:B * mb].reshape(B, mb).astype(np.int32)
    kp = torch.randn((L, pages, H, P, D)).to(torch.bfloat16)   # stale contents everywhere
    vp = torch.randn((L, pages, H, P, D)).to(torch.bfloat16)
    for b in range(B):
        for j in range(mb):
            kp[:, bt[b, j]] = K[:, b, :, j * P:(j + 1) * P]
            vp[:, bt[b, j]] = V[:, b, :, j * P:(j + 1) * P]
    return kp, vp, bt


def _from_pages(pool, bt, P):
    L, pages, H, _, D = pool.shape
    B, mb = bt.shape
    out = torch.empty((L, B, H, mb * P, D), dtype=pool.dtype)
    for b in range(B):
        for j in range(mb):
            out[:, b, :, j * P:(j + 1) * P] = pool[:, bt[b, j]]
    return out


@pytest.mark.parametrize("P", [16, 32, 64, 128])
def test_paged_equals_contiguous_and_the_oracle(rkv, P):
    w = Workload("pg", 2, 3, 2, 8, 128, (384, 250, 100), buffer=128, seed=95)
    x = make_inputs(w)
    cap = x["K"].shape[3]
    pad = (-cap) % P
    if pad:
        x = dict(x, K=torch.nn.functional.pad(x["K"], (0, 0, 0, pad)),
                 V=torch.nn.functional.pad(x["V"], (0, 0, 0, pad)))
    dev = torch.device("cuda")
    budgets_h = [384, 250, 100]
    budgets = torch.tensor(budgets_h, dtype=torch.int32, device=dev)
    ref = run_step(rkv, w, x, budgets=budgets, cluster_size=1)

    kp, vp, bt = _to_pages(x, P, spare=5, seed=P)
    L, B, H, capp, D = x["K"].shape
    kpd, vpd = kp.to(dev), vp.to(dev)
    btd = torch.from_numpy(bt).to(dev)
    cur = x["cur_len"].to(dev).clone()
    cfg = rkv.make_config(384, 128, 8, 128, 2, 8, 0.1)
    ws = torch.zeros(rkv.rkv_workspace_size(cfg, L, B, capp), dtype=torch.uint8, device=dev)
    freed = torch.full(bt.shape, -1, dtype=torch.int32, device=dev)
    n_freed = torch.full((B,), -1, dtype=torch.int32, device=dev)
    kept = torch.full((L, B, H, capp), -1, dtype=torch.int32, device=dev)
    scores = torch.full((L, B, H, 4, capp), float("nan"), dtype=torch.float32, device=dev)
    rkv.rkv_compress_step_paged(cfg, kpd, vpd, x["Q"].to(dev), cur, ws, btd, P, freed, n_freed,
                                budgets=budgets, kept_out=kept, scores_out=scores)
    torch.cuda.synchronize()
    assert rkv.rkv_workspace_status(ws) == 0
    assert cur.tolist() == budgets_h
    # bit-identical to the contiguous step (same arithmetic, other addresses)
    assert np.array_equal(kept.cpu().numpy(), ref["kept"][..., :capp])
    s_ref = ref["scores"][..., :capp]
    s_pg = scores.cpu().numpy()
    assert np.array_equal(np.nan_to_num(s_pg, nan=7.0).view(np.uint32),
                          np.nan_to_num(s_ref, nan=7.0).view(np.uint32))
    Kc = _from_pages(kpd.cpu(), bt, P)
    Vc = _from_pages(vpd.cpu(), bt, P)
    for b, bud in enumerate(budgets_h):
        assert torch.equal(Kc[:, b, :, :bud].view(torch.int16), ref["K"][:, b, :, :bud].cpu().view(torch.int16))
        assert torch.equal(Vc[:, b, :, :bud].view(torch.int16), ref["V"][:, b, :, :bud].cpu().view(torch.int16))
    verify(w, x, {"K": Kc, "V": Vc, "kept": kept.cpu().numpy(), "scores": s_pg},
           all_units(w), lambda b: budgets_h[b], lambda b: w.mix_lambda)
    # the pages given back, and the spare pages untouched
    nf = n_freed.cpu().tolist()
    fr = freed.cpu().numpy()
    for b, bud in enumerate(budgets_h):
        want = onp.freed_pages(bt[b], int(x["cur_len"][b]), bud, P)
        assert nf[b] == len(want) and fr[b, :nf[b]].tolist() == want
    spare = sorted(set(range(kp.shape[1])) - set(bt.ravel().tolist()))
    for pg in spare:
        assert torch.equal(kpd[:, pg].cpu().view(torch.int16), kp[:, pg].view(torch.int16))


def test_not_due_sequence_keeps_its_pages(rkv):
    w = Workload("pgnd", 1, 2, 2, 8, 128, (256,), seed=96)
    x = make_inputs(w)
    dev = torch.device("cuda")
    P = 64
    kp, vp, bt = _to_pages(x, P, spare=0, seed=3)
    L, B, H, cap, D = x["K"].shape
    kpd, vpd = kp.to(dev), vp.to(dev)
    cur = x["cur_len"].to(dev).clone()
    cur[1] -= 3
    cfg = rkv.make_config(256, 128, 8, 128, 2, 8, 0.1)
    ws = torch.zeros(rkv.rkv_workspace_size(cfg, L, B, cap), dtype=torch.uint8, device=dev)
    freed = torch.full(bt.shape, -1, dtype=torch.int32, device=dev)
    n_freed = torch.full((B,), -1, dtype=torch.int32, device=dev)
    rkv.rkv_compress_step_paged(cfg, kpd, vpd, x["Q"].to(dev), cur, ws,
                                torch.from_numpy(bt).to(dev), P, freed, n_freed)
    torch.cuda.synchronize()
    assert n_freed.tolist() == [2, 0]             # 384 rows -> 256: pages 4 and 5 of 6 -> 4
    assert freed[0, :2].tolist() == bt[0, 4:6].tolist()
    for j in range(bt.shape[1]):
        assert torch.equal(kpd[:, bt[1, j]].cpu().view(torch.int16), kp[:, bt[1, j]].view(torch.int16))
