"""GPU parity of the fused compression step (rkv_compress_step) against the
oracle, through the C ABI, on sizes the oracle finishes in seconds."""
import numpy as np
import pytest
import torch

import oracle
from rkv_synth import WORKLOADS, Workload, make_inputs
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rkv(cuda_device):
    from decode_kv_cache_head_b200 import build
    build.build()
    import decode_kv_cache_head_b200 as m
    return m


def run_step(rkv, w, x, lam=None, budgets=None, lambdas=None, cur_len=None, cluster_size=0,
             pool=0, red_mode=0):
    """Runs the fused step on copies of x's tensors; returns everything to compare."""
    dev = torch.device("cuda")
    K = x["K"].to(dev).clone()
    V = x["V"].to(dev).clone()
    Q = x["Q"].to(dev)
    L, B, H, cap, D = K.shape
    cur = (x["cur_len"] if cur_len is None else cur_len).to(dev).clone()
    cfg = rkv.make_config(w.budget_of(0), w.buffer, w.window, 128, w.n_kv_heads, w.n_q_heads,
                          w.mix_lambda if lam is None else lam, gqa_pool=pool,
                          redundancy_mode=red_mode)
    ws = torch.zeros(rkv.rkv_workspace_size(cfg, L, B, cap), dtype=torch.uint8, device=dev)
    kept = torch.full((L, B, H, cap), -1, dtype=torch.int32, device=dev)
    scores = torch.full((L, B, H, 4, cap), float("nan"), dtype=torch.float32, device=dev)
    rkv.rkv_compress_step(cfg, K, V, Q, cur, ws, budgets=budgets, lambdas=lambdas,
                          kept_out=kept, scores_out=scores, cluster_size=cluster_size)
    torch.cuda.synchronize()
    assert rkv.rkv_workspace_status(ws) == 0
    return {"K": K, "V": V, "cur_len": cur, "kept": kept.cpu().numpy(),
            "scores": scores.cpu().numpy()}


def verify(w, x, out, units, budget_of, lam_of, pool=0, due=None, red_mode=0):
    G = w.n_q_heads // w.n_kv_heads
    N_of = lambda b: int(x["cur_len"][b])
    due = due or (lambda b: True)
    units = [u for u in units if due(u[1])]
    orc = gc.oracle_for_units(x["K"], x["Q"], units, N_of, budget_of, lam_of, G, pool=pool,
                              red_mode=red_mode)
    und = []
    for i, (l, b, h) in enumerate(units):
        N, bud = N_of(b), budget_of(b)
        M = N - w.window
        s = out["scores"][l, b, h]
        gc.check_scores("M*I", s[0, :M], orc["I"][i, :M], scale=M)
        gc.check_scores("r", s[1, :M], orc["r"][i, :M])
        gc.check_scores("M*R", s[2, :M], orc["R"][i, :M], scale=M)
        kept = out["kept"][l, b, h, :bud]
        gc.check_kept_layout(kept, M, N, bud)
        und.append(gc.boundary_check(orc["Z"][i, :M], kept[: bud - w.window], bud - w.window))
        gc.check_compaction(x["K"][l, b, h], out["K"][l, b, h], kept, bud)
        gc.check_compaction(x["V"][l, b, h], out["V"][l, b, h], kept, bud)
    return float(np.mean(und)) if und else 0.0


def all_units(w):
    return [(l, b, h) for l in range(w.n_layers) for b in range(w.batch)
            for h in range(w.n_kv_heads)]


def test_single_layer_workload(rkv):
    """One layer, batch 1, 8 KV / 32 query heads, N = 1152 (budget 1024 + 128)."""
    w = WORKLOADS["single_layer"]
    x = make_inputs(w)
    out = run_step(rkv, w, x)
    und = verify(w, x, out, all_units(w), w.budget_of, lambda b: w.mix_lambda)
    assert und < 0.01
    assert out["cur_len"].tolist() == [w.budget_of(0)]


@pytest.mark.parametrize("cluster_size,budget", [(2, 512), (4, 1024), (8, 1024), (16, 1024),
                                                 (16, 4000)])
def test_cluster_sizes(rkv, cluster_size, budget):
    """Every CTA count per unit gives the same parity (rows per CTA up to 264)."""
    w = Workload("cs", 2, 1, 2, 8, 128, (budget,), seed=61)
    x = make_inputs(w)
    out = run_step(rkv, w, x, cluster_size=cluster_size)
    verify(w, x, out, all_units(w), w.budget_of, lambda b: w.mix_lambda)


def test_rows_per_cta_limit_is_reported(rkv):
    """Two CTAs for 1152 rows would need 576 rows each (> 512): refused on the host."""
    w = Workload("cs2", 1, 1, 2, 8, 128, (1024,), seed=61)
    x = make_inputs(w)
    with pytest.raises(rkv.RkvError) as e:
        run_step(rkv, w, x, cluster_size=2)
    assert e.value.status == -6


@pytest.mark.parametrize("lam", [0.0, 1.0])
@pytest.mark.parametrize("pool", [0, 1])
def test_ablation_extremes(rkv, lam, pool):
    """lambda = 0 / 1 and mean pooling over the GQA group (the pages' ablations)."""
    w = Workload("ab", 1, 1, 2, 8, 128, (512,), seed=62)
    x = make_inputs(w)
    out = run_step(rkv, w, x, lam=lam, pool=pool)
    verify(w, x, out, all_units(w), w.budget_of, lambda b: lam, pool=pool)


@pytest.mark.parametrize("red_mode", [0, 1], ids=["mean", "max"])
def test_group_of_five_and_ragged_lengths(rkv, red_mode):
    """Qwen-14B-like group (G = 5, 40 query columns padded to 48) and lengths that
    are not multiples of 16, several sequences per batch, in both redundancy modes."""
    w = Workload("g5", 2, 3, 2, 10, 128, (900, 1500, 333), buffer=97, seed=63)
    x = make_inputs(w)
    budgets = torch.tensor([w.budget_of(b) for b in range(3)], dtype=torch.int32, device="cuda")
    out = run_step(rkv, w, x, budgets=budgets, red_mode=red_mode)
    verify(w, x, out, all_units(w), w.budget_of, lambda b: w.mix_lambda, red_mode=red_mode)
    assert out["cur_len"].tolist() == [900, 1500, 333]


def test_per_sequence_budgets_lambdas_and_not_due(rkv):
    """Ragged budgets and lambdas; sequence 1 is below budget + buffer and must be
    left untouched, sequence 3 has compression disabled (budget 0)."""
    w = Workload("rg", 1, 4, 2, 8, 128, (512, 1024, 300, 200), seed=64)
    x = make_inputs(w)
    cur = x["cur_len"].clone()
    cur[1] -= 1                                   # one token short of due
    budgets = torch.tensor([512, 1024, 300, 0], dtype=torch.int32, device="cuda")
    lambdas = torch.tensor([0.1, 0.5, 0.0, 1.0], dtype=torch.float32, device="cuda")
    lam_h = [0.1, 0.5, 0.0, 1.0]
    out = run_step(rkv, w, x, budgets=budgets, lambdas=lambdas, cur_len=cur)
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
    out = run_step(rkv, w, x)
    assert out["kept"][0, 0, 0, :8].tolist() == list(range(40, 48))
    gc.check_compaction(x["K"][0, 0, 0], out["K"][0, 0, 0], out["kept"][0, 0, 0], 8)


def test_identical_keys_keep_the_oldest(rkv):
    """All keys equal: every Z ties, so the lowest indices survive (the tie rule)."""
    w = Workload("eq", 1, 1, 1, 4, 128, (200,), buffer=56, seed=66)
    x = make_inputs(w)
    x["K"][0, 0, 0, :256] = x["K"][0, 0, 0, 3]
    out = run_step(rkv, w, x)
    assert out["kept"][0, 0, 0, :200].tolist() == list(range(192)) + list(range(248, 256))


def test_deterministic(rkv):
    w = Workload("det", 4, 2, 2, 8, 128, (1024,), seed=67)
    x = make_inputs(w)
    a = run_step(rkv, w, x)
    b = run_step(rkv, w, x)
    assert np.array_equal(a["kept"], b["kept"])
    assert np.array_equal(a["scores"].view(np.uint32), b["scores"].view(np.uint32))
    assert torch.equal(a["K"].view(torch.int16), b["K"].view(torch.int16))
    assert torch.equal(a["V"].view(torch.int16), b["V"].view(torch.int16))


def test_second_call_is_a_no_op(rkv):
    """After compression cur_len = budget, so the next call finds nothing due."""
    w = Workload("noop", 1, 1, 2, 8, 128, (256,), seed=68)
    x = make_inputs(w)
    out = run_step(rkv, w, x)
    again = run_step(rkv, w, {"K": out["K"].cpu(), "V": out["V"].cpu(), "Q": x["Q"],
                              "cur_len": out["cur_len"].cpu()})
    assert torch.equal(again["K"], out["K"]) and torch.equal(again["V"], out["V"])


@pytest.mark.parametrize("lam", [0.1, 0.0, 1.0])
def test_max_redundancy_step(rkv, lam):
    """The step in MAX mode: tcgen05 similarity kernel, then the fused kernel.  Near
    duplicates make genuine near-ties under MAX; only decided tokens must agree."""
    w = Workload("mx", 2, 2, 2, 8, 128, (1024, 700), seed=69)
    x = make_inputs(w)
    budgets = torch.tensor([1024, 700], dtype=torch.int32, device="cuda")
    out = run_step(rkv, w, x, lam=lam, budgets=budgets, red_mode=1)
    und = verify(w, x, out, all_units(w), w.budget_of, lambda b: lam, red_mode=1)
    print(f"MAX mode lambda={lam}: undecided fraction {und:.4f}")
