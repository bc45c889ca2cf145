"""rkv_compress_step_noalloc, the step for callers that cannot allocate device
memory: a plugin inside a serving engine that keeps all GPU memory in its own
pool, or a decode loop in which an allocation (which may synchronise the
device) is not allowed.  Such a caller has no workspace to hand over, so the
library supplies a small fixed scratch array of its own.

Checked here, through the C ABI: two calls in a row on each launch shape (the
cluster kernel and the one-CTA-per-unit kernel), each compared with
rkv_compress_step on the same inputs and its device-side status read back with
rkv_noalloc_status; one call against the oracle; MAX redundancy and an
oversized batch rejected on the host; a bad per-sequence budget reported
through the status word.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from rkv_synth import Workload, make_inputs
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu

RKV_ERR_UNSUPPORTED, RKV_ERR_DEVICE_INPUT = -6, -9


@pytest.fixture(scope="module")
def libs(cuda_device):
    from decode_kv_cache_head_b200 import build
    build.build()
    import decode_kv_cache_head_b200 as rkv
    from decode_kv_cache_head_b200 import noalloc
    return rkv, noalloc


def _run(rkv, noalloc, fn, w, x, lambdas=None, budgets=None, cluster_size=0):
    dev = torch.device("cuda")
    K, V, Q = x["K"].to(dev).clone(), x["V"].to(dev).clone(), x["Q"].to(dev)
    cur = x["cur_len"].to(dev).clone()
    L, B, H, cap, D = K.shape
    cfg = rkv.make_config(w.budget_of(0), w.buffer, w.window, 128, w.n_kv_heads, w.n_q_heads,
                          w.mix_lambda)
    kept = torch.full((L, B, H, cap), -1, dtype=torch.int32, device=dev)
    scores = torch.zeros((L, B, H, 4, cap), dtype=torch.float32, device=dev)
    if fn == "workspace":
        ws = torch.zeros(rkv.rkv_workspace_size(cfg, L, B, cap), dtype=torch.uint8, device=dev)
        rkv.rkv_compress_step(cfg, K, V, Q, cur, ws, budgets=budgets, lambdas=lambdas,
                              kept_out=kept, scores_out=scores, cluster_size=cluster_size)
        status = rkv.rkv_workspace_status(ws)
    else:
        noalloc.rkv_compress_step_noalloc(cfg, K, V, Q, cur, budgets=budgets, lambdas=lambdas,
                                          kept_out=kept, scores_out=scores,
                                          cluster_size=cluster_size)
        status = noalloc.rkv_noalloc_status()
    torch.cuda.synchronize()
    return K, V, cur, kept.cpu().numpy(), scores.cpu().numpy(), status


CASES = [
    (Workload("na1", 2, 3, 2, 8, 128, (512, 700, 300), seed=91), [0.1, 0.5, 1.0]),
    (Workload("na2", 1, 2, 2, 10, 128, (900, 400), buffer=64, seed=92), [0.0, 0.1]),
]


@pytest.mark.parametrize("cluster_size", [0, 1], ids=["auto-cluster", "one-cta-per-unit"])
def test_noalloc_step_matches_the_workspace_step_on_two_calls_in_a_row(libs, cluster_size):
    rkv, noalloc = libs
    dev = torch.device("cuda")
    for w, lams in CASES:      # two calls in a row; the second sees the first's leftovers
        x = make_inputs(w)
        budgets = torch.tensor([w.budget_of(b) for b in range(w.batch)], dtype=torch.int32,
                               device=dev)
        lambdas = torch.tensor(lams, dtype=torch.float32, device=dev)
        Kr, Vr, cr, kr, sr, st_r = _run(rkv, noalloc, "workspace", w, x, lambdas, budgets,
                                        cluster_size)
        Kn, Vn, cn, kn, sn, st_n = _run(rkv, noalloc, "noalloc", w, x, lambdas, budgets,
                                        cluster_size)
        assert st_r == 0 and st_n == 0, (st_r, st_n)
        assert torch.equal(cn, cr)
        assert cn.tolist() == [w.budget_of(b) for b in range(w.batch)]
        for l in range(w.n_layers):
            for b in range(w.batch):
                N, bud = int(x["cur_len"][b]), w.budget_of(b)
                M = N - w.window
                for h in range(w.n_kv_heads):
                    np.testing.assert_array_equal(kn[l, b, h, :bud], kr[l, b, h, :bud])
                    gc.check_scores("M*I", sn[l, b, h, 0, :M], sr[l, b, h, 0, :M].astype(np.float64), scale=M)
                    gc.check_scores("r", sn[l, b, h, 1, :M], sr[l, b, h, 1, :M].astype(np.float64))
                    gc.check_scores("M*R", sn[l, b, h, 2, :M], sr[l, b, h, 2, :M].astype(np.float64), scale=M)
                    assert torch.equal(Kn[l, b, h, :bud].view(torch.int16),
                                       Kr[l, b, h, :bud].view(torch.int16))
                    assert torch.equal(Vn[l, b, h, :bud].view(torch.int16),
                                       Vr[l, b, h, :bud].view(torch.int16))


def test_noalloc_step_against_the_oracle(libs):
    rkv, noalloc = libs
    dev = torch.device("cuda")
    w, lams = CASES[0]
    x = make_inputs(w)
    budgets = torch.tensor([w.budget_of(b) for b in range(w.batch)], dtype=torch.int32, device=dev)
    lambdas = torch.tensor(lams, dtype=torch.float32, device=dev)
    K, V, cur, kept, scores, st = _run(rkv, noalloc, "noalloc", w, x, lambdas, budgets)
    assert st == 0
    G = w.n_q_heads // w.n_kv_heads
    units = [(l, b, h) for l in range(w.n_layers) for b in range(w.batch)
             for h in range(w.n_kv_heads)]
    orc = gc.oracle_for_units(x["K"], x["Q"], units, lambda b: int(x["cur_len"][b]),
                              w.budget_of, lambda b: lams[b], G)
    for i, (l, b, h) in enumerate(units):
        N, bud = int(x["cur_len"][b]), w.budget_of(b)
        M = N - w.window
        gc.check_scores("M*I", scores[l, b, h, 0, :M], orc["I"][i, :M], scale=M)
        gc.check_scores("M*R", scores[l, b, h, 2, :M], orc["R"][i, :M], scale=M)
        kp = kept[l, b, h, :bud]
        gc.check_kept_layout(kp, M, N, bud)
        gc.boundary_check(orc["Z"][i, :M], kp[: bud - w.window], bud - w.window)
        gc.check_compaction(x["K"][l, b, h], K[l, b, h], kp, bud)
        gc.check_compaction(x["V"][l, b, h], V[l, b, h], kp, bud)


def test_noalloc_step_reports_a_bad_device_side_budget(libs):
    rkv, noalloc = libs
    dev = torch.device("cuda")
    w, lams = CASES[0]
    x = make_inputs(w)
    # sequence 1's budget is below the window: only the device sees it; the step
    # skips that sequence, compresses the others and flags the status word
    bad = [w.budget_of(0), 4, w.budget_of(2)]
    budgets = torch.tensor(bad, dtype=torch.int32, device=dev)
    K, V, cur, kept, _, st = _run(rkv, noalloc, "noalloc", w, x, None, budgets)
    assert st == RKV_ERR_DEVICE_INPUT
    assert cur.tolist() == [w.budget_of(0), int(x["cur_len"][1]), w.budget_of(2)]
    assert torch.equal(K[:, 1].cpu().view(torch.int16), x["K"][:, 1].view(torch.int16))
    # the next good call starts from a clean status word
    budgets = torch.tensor([w.budget_of(b) for b in range(w.batch)], dtype=torch.int32, device=dev)
    *_, st = _run(rkv, noalloc, "noalloc", w, x, None, budgets)
    assert st == 0


def test_noalloc_step_rejects_what_its_scratch_cannot_hold(libs):
    rkv, noalloc = libs
    cfg = rkv.make_config(64, 16, 8, 128, 1, 4, 0.1)
    n = noalloc.RKV_NOALLOC_MAX_BATCH + 1
    arr = (ctypes.c_void_p * 1)(1 << 40)
    st = noalloc._f(ctypes.byref(cfg), 1, n, 128, arr, (ctypes.c_void_p * 1)(1 << 41),
                    (ctypes.c_void_p * 1)(1 << 42), None, None, 1 << 43, None, None)
    assert st == RKV_ERR_UNSUPPORTED
    # MAX redundancy keeps r of every unit in the workspace: not in the scratch
    cfg_max = rkv.make_config(64, 16, 8, 128, 1, 4, 0.1, redundancy_mode=rkv.RKV_RED_MAX)
    st = noalloc._f(ctypes.byref(cfg_max), 1, 2, 128, arr, (ctypes.c_void_p * 1)(1 << 41),
                    (ctypes.c_void_p * 1)(1 << 42), None, None, 1 << 43, None, None)
    assert st == RKV_ERR_UNSUPPORTED
