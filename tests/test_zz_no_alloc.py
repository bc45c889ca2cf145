"""rkv_compress_step_noalloc, the step for callers that cannot allocate device
memory (for instance a plugin inside a serving engine that keeps all GPU memory
in its own pool): two calls in a row, each compared with rkv_compress_step on
the same inputs.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from rkv_synth import Workload, make_inputs
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu


def _run(rkv, fn, w, x, lambdas=None, budgets=None):
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
                              kept_out=kept, scores_out=scores)
    else:
        from decode_kv_cache_head_b200 import noalloc
        noalloc.rkv_compress_step_noalloc(cfg, K, V, Q, cur, budgets=budgets, lambdas=lambdas,
                                          kept_out=kept, scores_out=scores)
    torch.cuda.synchronize()
    return K, V, cur, kept.cpu().numpy(), scores.cpu().numpy()


def test_noalloc_step_matches_the_workspace_step_on_two_calls_in_a_row(cuda_device):
    from decode_kv_cache_head_b200 import build
    build.build()
    import decode_kv_cache_head_b200 as rkv

    dev = torch.device("cuda")
    cases = [
        (Workload("na1", 2, 3, 2, 8, 128, (512, 700, 300), seed=91), [0.1, 0.5, 1.0]),
        (Workload("na2", 1, 2, 2, 10, 128, (900, 400), buffer=64, seed=92), [0.0, 0.1]),
    ]
    for w, lams in cases:      # two calls in a row; the second sees the first's leftovers
        x = make_inputs(w)
        budgets = torch.tensor([w.budget_of(b) for b in range(w.batch)], dtype=torch.int32,
                               device=dev)
        lambdas = torch.tensor(lams, dtype=torch.float32, device=dev)
        Kr, Vr, cr, kr, sr = _run(rkv, "workspace", w, x, lambdas, budgets)
        Kn, Vn, cn, kn, sn = _run(rkv, "noalloc", w, x, lambdas, budgets)
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


def test_noalloc_step_rejects_a_batch_beyond_its_scratch(cuda_device):
    from decode_kv_cache_head_b200 import build
    build.build()
    import decode_kv_cache_head_b200 as rkv
    from decode_kv_cache_head_b200 import noalloc

    cfg = rkv.make_config(64, 16, 8, 128, 1, 4, 0.1)
    n = noalloc.RKV_NOALLOC_MAX_BATCH + 1
    arr = (ctypes.c_void_p * 1)(1 << 40)
    st = noalloc._f(ctypes.byref(cfg), 1, n, 128, arr, (ctypes.c_void_p * 1)(1 << 41),
                    (ctypes.c_void_p * 1)(1 << 42), None, None, 1 << 43, None, None)
    assert st == -6
