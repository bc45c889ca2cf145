"""The seeded generator: shapes, reproducibility and the near-duplicate runs."""
import numpy as np
import torch

from rkv_synth import WORKLOADS, Workload, dup_runs, make_inputs


def test_dup_runs_structure():
    for seed in range(5):
        n = 1152
        runs = dup_runs(n, 0.3, seed)
        covered = np.zeros(n, dtype=int)
        for (p, s, L) in runs:
            assert 4 <= L <= 16
            assert s + L <= p and p + L <= n
            covered[p:p + L] += 1
        assert covered.max() == 1                       # destinations never overlap
        assert abs(covered.sum() / n - 0.3) < 0.02      # about 30% of positions


def test_make_inputs_shapes_and_copies():
    w = Workload("t", 2, 2, 2, 8, 128, (48, 40), dup_frac=(0.3,), seed=11)
    x = make_inputs(w)
    K, V, Q = x["K"], x["V"], x["Q"]
    assert K.shape == (2, 2, 2, w.cap, 128) and K.dtype == torch.bfloat16
    assert Q.shape == (2, 2, 8, w.window, 128)
    assert x["cur_len"].tolist() == [48 + 128, 40 + 128]
    n1 = 40 + 128
    assert torch.count_nonzero(K[:, 1, :, n1:]) == 0      # unused capacity is zero
    runs = dup_runs(n1, 0.3, seed=11 * 1_000_003 + 1)
    p, s, L = runs[0]
    a = K[0, 1, 0, p].float()
    b = K[0, 1, 0, s].float()
    cos = torch.dot(a, b) / (a.norm() * b.norm())
    assert cos > 0.99


def test_reproducible_and_layer_subsets():
    w = Workload("t", 3, 1, 2, 4, 128, (32,), seed=5)
    a = make_inputs(w)
    b = make_inputs(w, layers=[2])
    assert torch.equal(a["K"][2], b["K"][0]) and torch.equal(a["Q"][2], b["Q"][0])


def test_ar1_keys_are_correlated():
    w = Workload("t", 1, 1, 1, 4, 128, (512,), dup_frac=(0.0,), ar_rho=0.9, seed=3)
    k = make_inputs(w)["K"][0, 0, 0, :640].float()
    lag1 = (k[1:] * k[:-1]).mean() / (k * k).mean()
    assert 0.85 < float(lag1) < 0.95


def test_named_workloads():
    assert WORKLOADS["llama3_8b_step"].token_heads() == 32 * 8 * 1152
    assert WORKLOADS["qwen_14b_batched"].cap == 2176
    rag = WORKLOADS["ragged_batch"]
    assert set(rag.budgets) <= {512, 1024, 1536, 2048} and len(rag.budgets) == 64
