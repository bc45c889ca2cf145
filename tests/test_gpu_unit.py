"""GPU parity of the one-CTA-per-unit step kernel (cluster_size = 1) against the
oracle: the cases of the cluster kernel's tests plus the shapes this kernel
handles differently (one or many 128-row tiles, a ragged last tile, many
candidates per thread in the select, a runtime window, 64 query columns)."""
import numpy as np
import pytest
import torch

from rkv_synth import WORKLOADS, Workload, make_inputs
from tests import gpu_common as gc
from tests.test_gpu_step import all_units, run_step, verify

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rkv(cuda_device):
    from decode_kv_cache_head_b200 import build
    build.build()
    import decode_kv_cache_head_b200 as m
    return m


def test_single_layer_workload(rkv):
    w = WORKLOADS["single_layer"]
    x = make_inputs(w)
    out = run_step(rkv, w, x, cluster_size=1)
    und = verify(w, x, out, all_units(w), w.budget_of, lambda b: w.mix_lambda)
    assert und < 0.01
    assert out["cur_len"].tolist() == [w.budget_of(0)]


@pytest.mark.parametrize("budget,buffer", [(40, 16), (120, 8), (100, 28), (121, 8), (248, 8),
                                           (1000, 129), (3900, 100), (5000, 200)])
def test_tile_counts(rkv, budget, buffer):
    """N = 56 (one partial tile), 128 and 256 (whole tiles), 129 (a one-row tail),
    1129 (ragged), 4000 (16 candidates per thread) and 5200 (32 per thread)."""
    w = Workload("tiles", 1, 1, 2, 8, 128, (budget,), buffer=buffer, seed=71)
    x = make_inputs(w)
    out = run_step(rkv, w, x, cluster_size=1)
    verify(w, x, out, all_units(w), w.budget_of, lambda b: w.mix_lambda)


@pytest.mark.parametrize("lam", [0.0, 1.0])
@pytest.mark.parametrize("pool", [0, 1])
def test_ablation_extremes(rkv, lam, pool):
    w = Workload("ab", 1, 1, 2, 8, 128, (512,), seed=62)
    x = make_inputs(w)
    out = run_step(rkv, w, x, lam=lam, pool=pool, cluster_size=1)
    verify(w, x, out, all_units(w), w.budget_of, lambda b: lam, pool=pool)


@pytest.mark.parametrize("red_mode", [0, 1], ids=["mean", "max"])
@pytest.mark.parametrize("n_q,window", [(10, 8), (16, 8), (12, 4), (8, 3), (4, 16)])
def test_groups_and_windows(rkv, n_q, window, red_mode):
    """G = 5 (40 query columns padded to 48), G = 8 (64 columns), and windows other
    than 8 (the runtime-window kernel), with ragged lengths and several sequences, in
    both redundancy modes."""
    w = Workload("gw", 2, 3, 2, n_q, 128, (900, 1500, 333), buffer=97, window=window, seed=63)
    x = make_inputs(w)
    budgets = torch.tensor([w.budget_of(b) for b in range(3)], dtype=torch.int32, device="cuda")
    for pool in (0, 1):
        out = run_step(rkv, w, x, budgets=budgets, pool=pool, cluster_size=1, red_mode=red_mode)
        verify(w, x, out, all_units(w), w.budget_of, lambda b: w.mix_lambda, pool=pool,
               red_mode=red_mode)


def test_per_sequence_budgets_lambdas_and_not_due(rkv):
    w = Workload("rg", 1, 4, 2, 8, 128, (512, 1024, 300, 200), seed=64)
    x = make_inputs(w)
    cur = x["cur_len"].clone()
    cur[1] -= 1
    budgets = torch.tensor([512, 1024, 300, 0], dtype=torch.int32, device="cuda")
    lambdas = torch.tensor([0.1, 0.5, 0.0, 1.0], dtype=torch.float32, device="cuda")
    lam_h = [0.1, 0.5, 0.0, 1.0]
    out = run_step(rkv, w, x, budgets=budgets, lambdas=lambdas, cur_len=cur, cluster_size=1)
    x2 = dict(x, cur_len=cur)
    verify(w, x2, out, all_units(w), lambda b: int(budgets[b]), lambda b: lam_h[b],
           due=lambda b: b in (0, 2))
    assert out["cur_len"].tolist() == [512, int(cur[1]), 300, int(cur[3])]
    for b in (1, 3):
        assert torch.equal(out["K"][:, b].cpu(), x["K"][:, b])
        assert torch.equal(out["V"][:, b].cpu(), x["V"][:, b])


def test_budget_equal_to_window_keeps_only_the_window(rkv):
    w = Workload("kw", 1, 1, 1, 4, 128, (8,), buffer=40, seed=65)
    x = make_inputs(w)
    out = run_step(rkv, w, x, cluster_size=1)
    assert out["kept"][0, 0, 0, :8].tolist() == list(range(40, 48))
    gc.check_compaction(x["K"][0, 0, 0], out["K"][0, 0, 0], out["kept"][0, 0, 0], 8)


def test_identical_keys_keep_the_oldest(rkv):
    w = Workload("eq", 1, 1, 1, 4, 128, (200,), buffer=56, seed=66)
    x = make_inputs(w)
    x["K"][0, 0, 0, :256] = x["K"][0, 0, 0, 3]
    out = run_step(rkv, w, x, cluster_size=1)
    assert out["kept"][0, 0, 0, :200].tolist() == list(range(192)) + list(range(248, 256))


def test_zero_keys(rkv):
    """Zero rows: ||k|| clamps to 1e-12, khat = 0, similarity 0 with everything."""
    w = Workload("z", 1, 1, 2, 8, 128, (300,), seed=72)
    x = make_inputs(w)
    x["K"][0, 0, :, 5:40] = 0
    out = run_step(rkv, w, x, cluster_size=1)
    verify(w, x, out, all_units(w), w.budget_of, lambda b: w.mix_lambda)


def test_deterministic(rkv):
    w = Workload("det", 4, 2, 2, 8, 128, (1024,), seed=67)
    x = make_inputs(w)
    a = run_step(rkv, w, x, cluster_size=1)
    b = run_step(rkv, w, x, cluster_size=1)
    assert np.array_equal(a["kept"], b["kept"])
    assert np.array_equal(a["scores"].view(np.uint32), b["scores"].view(np.uint32))
    assert torch.equal(a["K"].view(torch.int16), b["K"].view(torch.int16))
    assert torch.equal(a["V"].view(torch.int16), b["V"].view(torch.int16))


@pytest.mark.parametrize("lam", [0.1, 0.0, 1.0])
def test_max_redundancy_step(rkv, lam):
    w = Workload("mx", 2, 2, 2, 8, 128, (1024, 700), seed=69)
    x = make_inputs(w)
    budgets = torch.tensor([1024, 700], dtype=torch.int32, device="cuda")
    out = run_step(rkv, w, x, lam=lam, budgets=budgets, red_mode=1, cluster_size=1)
    verify(w, x, out, all_units(w), w.budget_of, lambda b: lam, red_mode=1)


@pytest.mark.parametrize("red_mode", [0, 1], ids=["mean", "max"])
def test_longest_cache(rkv, red_mode):
    """The longest cache the unit kernel and the similarity kernel take: N = 7680 rows
    (60 tiles; 7672 candidates, 30 per thread in the select; one CTA per SM)."""
    w = Workload("longest", 1, 1, 2, 8, 128, (7552,), buffer=128, seed=79)
    assert w.cap == 7680
    x = make_inputs(w)
    out = run_step(rkv, w, x, red_mode=red_mode, cluster_size=1)
    verify(w, x, out, all_units(w), w.budget_of, lambda b: w.mix_lambda, red_mode=red_mode)
    assert out["cur_len"].tolist() == [7552]


def test_automatic_choice_at_many_units(rkv):
    """With one unit per SM or more the step picks this kernel by itself; the result
    is identical to forcing it."""
    w = Workload("auto", 19, 1, 8, 32, 128, (256,), seed=73)   # 152 units
    cfg = rkv.make_config(256, 128, 8, 128, 8, 32, 0.1)
    assert rkv.rkv_query_step_shape(cfg, 152, w.cap)[0] == 1
    assert rkv.rkv_query_step_shape(cfg, 8, w.cap)[0] > 1
    x = make_inputs(w)
    a = run_step(rkv, w, x)
    b = run_step(rkv, w, x, cluster_size=1)
    assert np.array_equal(a["kept"], b["kept"])
    assert np.array_equal(a["scores"].view(np.uint32), b["scores"].view(np.uint32))
    units = [(l, 0, h) for l in (0, 9, 18) for h in range(8)]
    verify(w, x, a, units, w.budget_of, lambda b: w.mix_lambda)
