"""The largest-first unit order changes only which units start first.

rkv_workspace_size includes room for one int32 per sequence, in which the plan kernel
orders the sequences by decreasing length; the batched kernels then take the units of
the longest sequences first.  A workspace short of exactly that room is accepted and the
units run in launch order.  On a batch of sequences of very different lengths, in both
redundancy modes, the two runs must give bit-identical caches, kept indices and scores,
and the ordered run is checked against the oracle on sampled units.
"""
import numpy as np
import pytest
import torch

from rkv_synth import Workload, make_inputs
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rkv(cuda_device):
    from decode_kv_cache_head_b200 import build
    build.build()
    import decode_kv_cache_head_b200 as m
    return m


def _order_room(batch):
    return (batch * 4 + 255) // 256 * 256


def _run(rkv, w, x, red_mode, shrink):
    dev = torch.device("cuda")
    K, V, Q = x["K"].to(dev).clone(), x["V"].to(dev).clone(), x["Q"].to(dev)
    cur = x["cur_len"].to(dev).clone()
    L, B, H, cap, _ = K.shape
    cfg = rkv.make_config(w.budget_of(0), w.buffer, w.window, 128, w.n_kv_heads, w.n_q_heads,
                          w.mix_lambda, redundancy_mode=red_mode)
    size = rkv.rkv_workspace_size(cfg, L, B, cap) - (_order_room(B) if shrink else 0)
    ws = torch.zeros(size, dtype=torch.uint8, device=dev)
    budgets = torch.tensor([w.budget_of(b) for b in range(B)], dtype=torch.int32, device=dev)
    kept = torch.full((L, B, H, cap), -1, dtype=torch.int32, device=dev)
    scores = torch.zeros((L, B, H, 4, cap), dtype=torch.float32, device=dev)
    rkv.rkv_compress_step(cfg, K, V, Q, cur, ws, budgets=budgets, kept_out=kept,
                          scores_out=scores, cluster_size=1)
    torch.cuda.synchronize()
    assert rkv.rkv_workspace_status(ws) == 0
    return K, V, cur, kept, scores


@pytest.mark.parametrize("red_mode", [0, 1], ids=["mean", "max"])
def test_ordered_and_launch_order_runs_are_bit_identical(rkv, red_mode):
    # lengths from 1 to 17 tiles, shuffled so that the launch order is not sorted already
    budgets = (1024, 160, 2048, 512, 1536, 256, 896, 2000)
    w = Workload("order", 2, len(budgets), 4, 16, 128, budgets, seed=97)
    x = make_inputs(w)
    a = _run(rkv, w, x, red_mode, shrink=False)
    b = _run(rkv, w, x, red_mode, shrink=True)
    for ta, tb in zip(a, b):
        if ta.dtype == torch.bfloat16:
            assert torch.equal(ta.view(torch.int16), tb.view(torch.int16))
        else:
            assert torch.equal(ta, tb)
    K, V, cur, kept, scores = a
    G = w.n_q_heads // w.n_kv_heads
    units = [(l, s, h) for l in range(w.n_layers) for s in (0, 1, 2, 5) for h in range(w.n_kv_heads)]
    orc = gc.oracle_for_units(x["K"], x["Q"], units, lambda s: int(x["cur_len"][s]), w.budget_of,
                              lambda s: w.mix_lambda, G, red_mode=red_mode)
    kept, scores = kept.cpu().numpy(), scores.cpu().numpy()
    for i, (l, s, h) in enumerate(units):
        N, bud = int(x["cur_len"][s]), w.budget_of(s)
        M = N - w.window
        gc.check_scores("M*I", scores[l, s, h, 0, :M], orc["I"][i, :M], scale=M)
        gc.check_scores("M*R", scores[l, s, h, 2, :M], orc["R"][i, :M], scale=M)
        kp = kept[l, s, h, :bud]
        gc.check_kept_layout(kp, M, N, bud)
        gc.boundary_check(orc["Z"][i, :M], kp[: bud - w.window], bud - w.window)
        gc.check_compaction(x["K"][l, s, h], K[l, s, h], kp, bud)
        gc.check_compaction(x["V"][l, s, h], V[l, s, h], kp, bud)
