"""Pins of the oracle's shared (cross-head / cross-rank) selection: one kept set
per (sequence, layer), chosen by the sum over the KV heads of their joint
scores (the tensor-parallel ranks' all-reduce of eviction scores, hysenlabs
write-up, decode-time section).  Each pin fixes the result from something other
than the function itself: brute force, the per-head definition it reduces to,
exact scalings and symmetries."""
import itertools

import numpy as np
import pytest

import torch

import oracle
from oracle import rkv_oracle_np as onp
from rkv_synth import bf16_bits


def _heads(seed, H, N, G=4, w=8, D=128):
    g = torch.Generator().manual_seed(seed)
    k = bf16_bits(torch.randn((H, N, D), generator=g).to(torch.bfloat16))
    q = bf16_bits(torch.randn((H, G, w, D), generator=g).to(torch.bfloat16))
    return q, k


def _brute(Zsum, N, budget):
    """Every k-subset of the candidates: the best by sum, ties by the lexicographically
    smallest index tuple (ascending) -- the rule (score desc, index asc) picks it."""
    M = Zsum.shape[0]
    kk = budget - (N - M)
    best, best_set = None, None
    for s in itertools.combinations(range(M), kk):
        v = sum(Zsum[i] for i in s)
        if best is None or v > best + 1e-15:
            best, best_set = v, s
    return np.array(list(best_set) + list(range(M, N)), dtype=np.int32)


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_on_tiny_inputs(seed):
    g = np.random.default_rng(100 + seed)
    H, N, budget = 3, 11, 7
    M = N - 2
    Z = g.normal(size=(H, M))
    Zsum, kept = oracle.shared_select(Z, N, budget)
    np.testing.assert_allclose(Zsum, Z[0] + Z[1] + Z[2], rtol=0, atol=1e-15)
    assert kept.tolist() == _brute(Zsum, N, budget).tolist()


def test_sum_not_max_nor_per_head():
    """A head that alone prefers token 0 loses to two heads preferring token 1."""
    Z = np.array([[5.0, 0.0, -1.0],
                  [0.0, 3.0, -1.0],
                  [0.0, 3.0, -1.0]])
    _, kept = oracle.shared_select(Z, 4, 2)     # M = 3, w = 1, keep 1 candidate
    assert kept.tolist() == [1, 3]


def test_one_head_is_the_per_head_step():
    q, k = _heads(7, 1, 300)
    out = oracle.shared_units(q, k, 300, 200, 0.1)
    assert out["kept_shared"].tolist() == out["kept"][0, :200].tolist()
    np.testing.assert_array_equal(out["Zsum"], out["Z"][0, :292])


def test_identical_heads_keep_what_one_head_keeps():
    """H copies of one head: Zsum = H * Z exactly (powers of two) keeps the same set."""
    q, k = _heads(8, 1, 260)
    q4, k4 = np.repeat(q, 4, axis=0), np.repeat(k, 4, axis=0)
    out = oracle.shared_units(q4, k4, 260, 130, 0.1)
    np.testing.assert_array_equal(out["Zsum"], 4.0 * out["Z"][0, :252])
    assert out["kept_shared"].tolist() == out["kept"][0, :130].tolist()


def test_head_order_and_rank_split():
    """Permuting heads, or summing two ranks' partial sums first (the all-reduce),
    keeps the set: only float rounding differs, so only exact near-ties may move."""
    q, k = _heads(9, 8, 400)
    out = oracle.shared_units(q, k, 400, 256, 0.1, n_threads=4)
    M = 392
    Z = out["Z"][:, :M]
    perm = np.random.default_rng(1).permutation(8)
    _, kp = oracle.shared_select(Z[perm], 400, 256)
    split = np.stack([Z[:4].sum(0), Z[4:].sum(0)])
    _, ks = oracle.shared_select(split, 400, 256)
    assert kp.tolist() == out["kept_shared"].tolist()
    assert ks.tolist() == out["kept_shared"].tolist()


def test_numpy_twin_agrees():
    q, k = _heads(10, 5, 333, G=5)
    out = oracle.shared_units(q, k, 333, 200, 0.3)
    zs, kept = onp.shared_select(out["Z"][:, :325], 333, 200)
    np.testing.assert_allclose(zs, out["Zsum"], rtol=1e-14, atol=1e-18)
    assert kept.tolist() == out["kept_shared"].tolist()


def test_shared_set_invariants():
    q, k = _heads(11, 8, 600)
    out = oracle.shared_units(q, k, 600, 300, 0.1, n_threads=4)
    kept = out["kept_shared"]
    assert len(kept) == 300 and np.all(np.diff(kept) > 0)
    assert kept[-8:].tolist() == list(range(592, 600))
    # every kept candidate scores at least as high as every evicted one
    Zs = out["Zsum"]
    ev = np.setdiff1d(np.arange(592), kept[:-8])
    assert Zs[kept[:-8]].min() >= Zs[ev].max()
