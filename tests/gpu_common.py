"""Helpers of the GPU parity tests: run the oracle on the same bf16 bits the
CUDA path read, and compare with the acceptance rules of the step:

* scores: M*I, M*R and r within rtol 1e-3 / atol 1e-5 (I and R are
  distributions over M ~ 10^3 candidates, so they are compared on the
  unit-mean scale M*I, M*R);
* kept sets: every candidate whose oracle M*Z lies more than 1e-4 from the
  oracle's k-th / (k+1)-th boundary midpoint is on the same side;
* exactly `budget` rows kept, ascending, the window included;
* compacted K/V bit-exact given the GPU's own kept indices.
"""
import os

import numpy as np
import torch

import oracle
from rkv_synth import bf16_bits

RTOL, ATOL, MARGIN = 1e-3, 1e-5, 1e-4


def n_threads():
    return max(1, os.cpu_count() or 1)


def oracle_for_units(K, Q, units, N_of, budget_of, lam_of, G, red_mode=oracle.RED_MEAN,
                     pool=oracle.POOL_MAX):
    """units: list of (l, b, h).  K [L,B,H,cap,D], Q [L,B,Hq,w,D] (any device)."""
    kb = bf16_bits(K)
    qb = bf16_bits(Q)
    q = np.stack([qb[l, b, h * G:(h + 1) * G] for (l, b, h) in units])
    k = np.stack([kb[l, b, h] for (l, b, h) in units])
    N = np.array([N_of(b) for (_, b, _) in units], dtype=np.int32)
    bud = np.array([budget_of(b) for (_, b, _) in units], dtype=np.int32)
    lam = np.array([lam_of(b) for (_, b, _) in units], dtype=np.float64)
    return oracle.units(q, k, N, bud, lam, red_mode=red_mode, pool=pool, n_threads=n_threads())


def boundary_check(Z, kept_cand, kk):
    """Z: oracle scores [M]; kept_cand: GPU-kept candidate indices.  Returns the
    undecided fraction; asserts every decided candidate is on the oracle's side."""
    M = Z.shape[0]
    sel = np.zeros(M, dtype=bool)
    sel[np.asarray(kept_cand, dtype=np.int64)] = True
    if kk <= 0:
        assert not sel.any()
        return 0.0
    if kk >= M:
        assert sel.all()
        return 0.0
    order = np.lexsort((np.arange(M), -Z))
    tau = 0.5 * (Z[order[kk - 1]] + Z[order[kk]])
    decided = np.abs(M * Z - M * tau) > MARGIN
    want = Z > tau
    bad = np.nonzero(decided & (sel != want))[0]
    assert bad.size == 0, f"{bad.size} decided candidates on the wrong side, e.g. {bad[:5]}"
    return float((~decided).mean())


def check_scores(name, got, want, scale=1.0):
    np.testing.assert_allclose(np.asarray(got, dtype=np.float64) * scale, want * scale,
                               rtol=RTOL, atol=ATOL, err_msg=name)


def check_kept_layout(kept, M, N, budget):
    kept = np.asarray(kept)
    assert kept.shape[0] == budget
    assert np.all(np.diff(kept) > 0), "kept indices must be strictly ascending"
    assert list(kept[budget - (N - M):]) == list(range(M, N)), "window must be kept"
    assert kept.min() >= 0 and kept.max() < N


def check_compaction(before, after, kept, budget):
    """before/after: [cap, D] bf16 tensors of one head; kept: [budget]."""
    b = before.view(torch.int16).cpu()
    a = after.view(torch.int16).cpu()
    idx = torch.as_tensor(np.asarray(kept[:budget], dtype=np.int64))
    assert torch.equal(a[:budget], b[idx]), "compacted rows differ from the gathered rows"
