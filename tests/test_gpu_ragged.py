"""rkv_compress_step_ragged: caches with per-sequence capacities.

Each sequence's [Hkv][cap_b][128] block sits at its own row of a per-layer
pool, so a sequence with a small budget holds only budget + buffer rows.
Checked against the oracle on every unit of a batch whose capacities run from
640 to 2176 rows (with slack rows and gaps between blocks, which must stay
untouched), in both redundancy modes; at the full ragged-batch size (64
sequences x 32 layers, blocks packed tight) the result must be bit-identical
to the uniform-layout step on the same rows, and sampled units are checked
against the oracle; a block that does not fit its pool is reported through
the workspace status and left alone.
"""
import numpy as np
import pytest
import torch

import oracle
from rkv_synth import WORKLOADS, Workload, make_inputs, pack_ragged, unpack_ragged
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rkv(cuda_device):
    from decode_kv_cache_head_b200 import build
    build.build()
    import decode_kv_cache_head_b200 as m
    return m


def _pool_with_gaps(X, caps, gaps, fill):
    """[L,B,H,cap,D] -> pool [L, rows, D] with `gaps[b]` filler rows before block b."""
    L, B, H, _, D = X.shape
    parts, rows, r = [], [], 0
    for b in range(B):
        if gaps[b]:
            parts.append(torch.full((L, gaps[b], D), fill, dtype=X.dtype, device=X.device))
            r += gaps[b]
        rows.append(r)
        parts.append(X[:, b, :, :caps[b]].reshape(L, H * caps[b], D))
        r += H * caps[b]
    return torch.cat(parts, dim=1).contiguous(), rows


def _run_ragged(rkv, w, x, caps, gaps, lam_list, red_mode=0, with_outputs=True):
    dev = torch.device("cuda")
    Kd, Vd = x["K"].to(dev), x["V"].to(dev)
    Kp, rows = _pool_with_gaps(Kd, caps, gaps, 0.5)
    Vp, _ = _pool_with_gaps(Vd, caps, gaps, -0.5)
    Q, cur = x["Q"].to(dev), x["cur_len"].to(dev).clone()
    L, B, H = w.n_layers, w.batch, w.n_kv_heads
    max_cap = max(caps)
    cfg = rkv.make_config(w.budget_of(0), w.buffer, w.window, 128, H, w.n_q_heads,
                          w.mix_lambda, redundancy_mode=red_mode)
    budgets = torch.tensor([w.budget_of(b) for b in range(B)], dtype=torch.int32, device=dev)
    lambdas = torch.tensor(lam_list, dtype=torch.float32, device=dev)
    seq_row = torch.tensor(rows, dtype=torch.int64, device=dev)
    seq_cap = torch.tensor(caps, dtype=torch.int32, device=dev)
    ws = torch.zeros(rkv.rkv_workspace_size(cfg, L, B, max_cap), dtype=torch.uint8, device=dev)
    kept = scores = None
    if with_outputs:
        kept = torch.full((L, B, H, max_cap), -1, dtype=torch.int32, device=dev)
        scores = torch.zeros((L, B, H, 4, max_cap), dtype=torch.float32, device=dev)
    K0, V0 = Kp.clone(), Vp.clone()
    rkv.rkv_compress_step_ragged(cfg, Kp, Vp, Q, cur, ws, seq_row, seq_cap, max_cap,
                                 budgets=budgets, lambdas=lambdas, kept_out=kept,
                                 scores_out=scores)
    torch.cuda.synchronize()
    return dict(K=Kp, V=Vp, K0=K0, V0=V0, rows=rows, cur=cur, kept=kept, scores=scores,
                status=rkv.rkv_workspace_status(ws))


def _block(P, rows, b, h, cap):
    r0 = rows[b] + h * cap
    return P[:, r0:r0 + cap]


@pytest.mark.parametrize("red_mode", [0, 1], ids=["mean", "max"])
def test_ragged_capacities_every_unit_against_the_oracle(rkv, red_mode):
    budgets = (512, 2048, 896, 1536, 1024, 300, 1920, 640)
    w = Workload("ragged_small", 2, len(budgets), 4, 16, 128, budgets, seed=41)
    x = make_inputs(w)
    slack = [0, 0, 16, 64, 5, 0, 33, 128]         # capacity beyond N (rows never read)
    gaps = [0, 7, 0, 128, 3, 0, 1, 0]              # filler rows between blocks
    caps = [w.budget_of(b) + w.buffer + slack[b] for b in range(w.batch)]
    lam_list = [(0.0, 0.1, 1.0)[b % 3] for b in range(w.batch)]
    out = _run_ragged(rkv, w, x, caps, gaps, lam_list, red_mode)
    assert out["status"] == 0
    assert out["cur"].tolist() == list(budgets)
    G = w.n_q_heads // w.n_kv_heads
    units = [(l, b, h) for l in range(w.n_layers) for b in range(w.batch)
             for h in range(w.n_kv_heads)]
    orc = gc.oracle_for_units(x["K"], x["Q"], units, lambda b: int(x["cur_len"][b]),
                              w.budget_of, lambda b: lam_list[b], G, red_mode=red_mode)
    kept, sc = out["kept"].cpu().numpy(), out["scores"].cpu().numpy()
    und = []
    for i, (l, b, h) in enumerate(units):
        N, bud = int(x["cur_len"][b]), w.budget_of(b)
        M = N - w.window
        gc.check_scores("M*I", sc[l, b, h, 0, :M], orc["I"][i, :M], scale=M)
        gc.check_scores("r", sc[l, b, h, 1, :M], orc["r"][i, :M])
        gc.check_scores("M*R", sc[l, b, h, 2, :M], orc["R"][i, :M], scale=M)
        kp = kept[l, b, h, :bud]
        gc.check_kept_layout(kp, M, N, bud)
        und.append(gc.boundary_check(orc["Z"][i, :M], kp[:bud - w.window], bud - w.window))
        for name in ("K", "V"):
            before = _block(out[name + "0"], out["rows"], b, h, caps[b])[l]
            after = _block(out[name], out["rows"], b, h, caps[b])[l]
            gc.check_compaction(before, after, kp, bud)
            # rows past N (slack) are never written
            assert torch.equal(after[N:].view(torch.int16), before[N:].view(torch.int16))
    # filler rows between the blocks are never written
    for b in range(w.batch):
        if gaps[b]:
            r1 = out["rows"][b]
            for name in ("K", "V"):
                assert torch.equal(out[name][:, r1 - gaps[b]:r1].view(torch.int16),
                                   out[name + "0"][:, r1 - gaps[b]:r1].view(torch.int16))
    print(f"ragged ({'max' if red_mode else 'mean'}): undecided fraction {np.mean(und):.4f}")


def test_ragged_batch_full_size_matches_the_uniform_layout(rkv):
    w = WORKLOADS["ragged_batch"]
    dev = torch.device("cuda")
    x = make_inputs(w, device="cuda")
    B, H, L = w.batch, w.n_kv_heads, w.n_layers
    caps = [w.budget_of(b) + w.buffer for b in range(B)]
    lam_list = [(0.0, 0.1, 1.0)[b % 3] for b in range(B)]
    # the ragged step, blocks packed tight (the bench's layout), no optional outputs
    Kp, Vp = pack_ragged(x["K"], caps), pack_ragged(x["V"], caps)
    rows = [0]
    for c in caps[:-1]:
        rows.append(rows[-1] + H * c)
    cfg = rkv.make_config(w.budget_of(0), w.buffer, w.window, 128, H, w.n_q_heads, w.mix_lambda)
    budgets = torch.tensor([w.budget_of(b) for b in range(B)], dtype=torch.int32, device=dev)
    lambdas = torch.tensor(lam_list, dtype=torch.float32, device=dev)
    seq_row = torch.tensor(rows, dtype=torch.int64, device=dev)
    seq_cap = torch.tensor(caps, dtype=torch.int32, device=dev)
    ws = torch.zeros(rkv.rkv_workspace_size(cfg, L, B, max(caps)), dtype=torch.uint8, device=dev)
    cur_r = x["cur_len"].clone()
    rkv.rkv_compress_step_ragged(cfg, Kp, Vp, x["Q"], cur_r, ws, seq_row, seq_cap, max(caps),
                                 budgets=budgets, lambdas=lambdas)
    torch.cuda.synchronize()
    assert rkv.rkv_workspace_status(ws) == 0
    # the uniform step on the same rows, with kept sets and scores for the oracle check
    K, V, cur_u = x["K"].clone(), x["V"].clone(), x["cur_len"].clone()
    cap = w.cap
    kept = torch.full((L, B, H, cap), -1, dtype=torch.int32, device=dev)
    scores = torch.zeros((L, B, H, 4, cap), dtype=torch.float32, device=dev)
    ws_u = torch.zeros(rkv.rkv_workspace_size(cfg, L, B, cap), dtype=torch.uint8, device=dev)
    rkv.rkv_compress_step(cfg, K, V, x["Q"], cur_u, ws_u, budgets=budgets, lambdas=lambdas,
                          kept_out=kept, scores_out=scores)
    torch.cuda.synchronize()
    assert rkv.rkv_workspace_status(ws_u) == 0
    assert torch.equal(cur_r, cur_u)
    assert torch.equal(pack_ragged(K, caps).view(torch.int16), Kp.view(torch.int16))
    assert torch.equal(pack_ragged(V, caps).view(torch.int16), Vp.view(torch.int16))
    del Kp, Vp
    # sampled units of the (identical) result against the oracle
    rng = np.random.default_rng(44)
    all_u = [(l, b, h) for l in range(L) for b in range(B) for h in range(H)]
    units = [all_u[i] for i in sorted(rng.choice(len(all_u), size=24, replace=False))]
    G = w.n_q_heads // H
    sub_K = torch.stack([x["K"][l, b, h].cpu() for (l, b, h) in units])
    sub_Q = torch.stack([x["Q"][l, b, h * G:(h + 1) * G].cpu() for (l, b, h) in units])
    orc = gc.oracle_for_units(sub_K[None, :, None], sub_Q[None],
                              [(0, i, 0) for i in range(len(units))],
                              lambda i: int(x["cur_len"][units[i][1]]),
                              lambda i: w.budget_of(units[i][1]),
                              lambda i: lam_list[units[i][1]], G)
    kept_h, sc = kept.cpu().numpy(), scores.cpu().numpy()
    for i, (l, b, h) in enumerate(units):
        N, bud = int(x["cur_len"][b]), w.budget_of(b)
        M = N - w.window
        gc.check_scores("M*I", sc[l, b, h, 0, :M], orc["I"][i, :M], scale=M)
        gc.check_scores("M*R", sc[l, b, h, 2, :M], orc["R"][i, :M], scale=M)
        kp = kept_h[l, b, h, :bud]
        gc.check_kept_layout(kp, M, N, bud)
        gc.boundary_check(orc["Z"][i, :M], kp[:bud - w.window], bud - w.window)
        gc.check_compaction(x["K"][l, b, h], K[l, b, h], kp, bud)
        gc.check_compaction(x["V"][l, b, h], V[l, b, h], kp, bud)


def test_ragged_block_outside_the_pool_is_reported_and_skipped(rkv):
    budgets = (300, 400)
    w = Workload("ragged_bad", 1, 2, 2, 8, 128, budgets, seed=43)
    x = make_inputs(w)
    dev = torch.device("cuda")
    caps = [w.budget_of(b) + w.buffer for b in range(2)]
    Kp, Vp = pack_ragged(x["K"].to(dev), caps), pack_ragged(x["V"].to(dev), caps)
    K0, V0 = Kp.clone(), Vp.clone()
    rows = [0, 2 * caps[0]]
    cfg = rkv.make_config(300, w.buffer, w.window, 128, 2, 8, 0.1)
    budgets = torch.tensor(list(budgets), dtype=torch.int32, device=dev)
    # sequence 1 claims one row more than the pool has
    seq_row = torch.tensor([rows[0], rows[1] + 1], dtype=torch.int64, device=dev)
    seq_cap = torch.tensor(caps, dtype=torch.int32, device=dev)
    cur = x["cur_len"].to(dev).clone()
    ws = torch.zeros(rkv.rkv_workspace_size(cfg, 1, 2, max(caps)), dtype=torch.uint8, device=dev)
    rkv.rkv_compress_step_ragged(cfg, Kp, Vp, x["Q"].to(dev), cur, ws, seq_row, seq_cap,
                                 max(caps), budgets=budgets)
    torch.cuda.synchronize()
    assert rkv.rkv_workspace_status(ws) == -9        # RKV_ERR_DEVICE_INPUT
    assert cur.tolist() == [300, int(x["cur_len"][1])]
    r1 = rows[1]
    assert torch.equal(Kp[:, r1:].view(torch.int16), K0[:, r1:].view(torch.int16))
    assert torch.equal(Vp[:, r1:].view(torch.int16), V0[:, r1:].view(torch.int16))
    assert not torch.equal(Kp[:, :r1].view(torch.int16), K0[:, :r1].view(torch.int16))
