"""Pins of the CPU oracle to facts outside itself.

Each test pins the oracle (both the C loops and the NumPy twin) to something
the R-KV pages or the mathematics fix: hand-derived closed forms, brute force
over every k-subset, library routines in special cases, and invariants.  The
cases are chosen so that a plausible slip -- a dropped 1/sqrt(D), a missing
causal mask, mean instead of max over the GQA group, a diagonal left in the
similarity, N instead of N-1, a flipped sign in Z, a wrong tie rule -- fails
at least one of them.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import rkv_oracle_np as onp

IMPLS = {
    "c": oracle,
    "numpy": onp,
}


def bits(x) -> np.ndarray:
    """float array -> bf16 bit patterns; asserts the values are bf16-exact."""
    t = torch.as_tensor(np.asarray(x, dtype=np.float32))
    b = t.to(torch.bfloat16)
    assert torch.equal(b.to(torch.float32), t), "test values must be exact in bf16"
    return b.view(torch.int16).numpy().view(np.uint16)


def rand_bits(rng, shape, scale=1.0):
    x = torch.as_tensor(rng.standard_normal(shape).astype(np.float32) * scale)
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def E(i, D, a=1.0):
    v = np.zeros(D, dtype=np.float32)
    v[i] = a
    return v


# --------------------------------------------------------------------------
# Importance
# --------------------------------------------------------------------------

@pytest.mark.parametrize("impl", IMPLS)
def test_importance_worked_example_scale_and_max_pool(impl):
    """G=2 heads, w=1, D=4, N=3 (M=2): logits q.k/sqrt(4).

    Head 0 (q=(2,0,0,0)) scores keys (1,0,0) -> p = (e,1,1)/(e+2); head 1
    (q=0) scores all keys 0 -> p = (1,1,1)/3.  Max over heads gives
    (e/(e+2), 1/3); mean gives ((e/(e+2)+1/3)/2, (1/(e+2)+1/3)/2).
    """
    D = 4
    q = bits([[E(0, D, 2.0)], [np.zeros(D)]])            # [G=2, w=1, D]
    k = bits([E(0, D), E(1, D), E(2, D)])                 # N=3
    e = math.e
    ihat_max = np.array([e / (e + 2), 1 / 3])
    ihat_mean = np.array([(e / (e + 2) + 1 / 3) / 2, (1 / (e + 2) + 1 / 3) / 2])
    got_max = IMPLS[impl].importance(q, k, 3, oracle.POOL_MAX)
    got_mean = IMPLS[impl].importance(q, k, 3, oracle.POOL_MEAN)
    np.testing.assert_allclose(got_max, ihat_max / ihat_max.sum(), rtol=1e-14)
    np.testing.assert_allclose(got_mean, ihat_mean / ihat_mean.sum(), rtol=1e-14)
    # without the 1/sqrt(D) scale head 0 would give e^2/(e^2+2): clearly different
    unscaled = np.array([e * e / (e * e + 2), 1 / 3])
    assert abs(got_max[0] - unscaled[0] / unscaled.sum()) > 1e-2


@pytest.mark.parametrize("impl", IMPLS)
def test_importance_causal_mask(impl):
    """G=1, w=2, D=4, N=4 (M=2).  Query 0 sits at position 2 and must not see key 3.

    q0=(2,0,0,2) scores keys k0=e0 -> 1, k1=e1 -> 0, k2=e2 -> 0, k3=e3 -> 1.
    With the mask query 0 sees keys 0..2: p = (e,1,1)/(e+2).  Query 1 (q=0)
    sees keys 0..3: p = 1/4 each.
    """
    D = 4
    q = bits([[E(0, D, 2.0) + E(3, D, 2.0), np.zeros(D)]])
    k = bits([E(0, D), E(1, D), E(2, D), E(3, D)])
    e = math.e
    a = np.array([(e / (e + 2) + 0.25) / 2, (1 / (e + 2) + 0.25) / 2])
    got = IMPLS[impl].importance(q, k, 4, oracle.POOL_MAX)
    np.testing.assert_allclose(got, a / a.sum(), rtol=1e-14)
    a_nomask = np.array([(e / (2 * e + 2) + 0.25) / 2, (1 / (2 * e + 2) + 0.25) / 2])
    assert abs(got[0] - a_nomask[0] / a_nomask.sum()) > 1e-3


@pytest.mark.parametrize("impl", IMPLS)
def test_importance_zero_queries_is_uniform(impl):
    """Q = 0: every candidate gets (1/w) sum_j 1/(M+j+1) -> I = 1/M exactly."""
    rng = np.random.default_rng(1)
    G, w, D, N = 3, 4, 16, 40
    q = bits(np.zeros((G, w, D)))
    k = rand_bits(rng, (N, D))
    got = IMPLS[impl].importance(q, k, N)
    np.testing.assert_allclose(got, np.full(N - w, 1.0 / (N - w)), rtol=1e-13)


@pytest.mark.parametrize("impl", IMPLS)
def test_importance_matches_library_attention(impl):
    """Attention probabilities come from torch's scaled_dot_product_attention.

    With V = identity, SDPA returns the attention-probability rows themselves
    (default scale 1/sqrt(D)); query j of the window may attend to keys
    0..M+j.  The window mean and the GQA max are then taken on those rows.
    """
    rng = np.random.default_rng(7)
    G, w, D, N = 4, 8, 128, 96
    M = N - w
    q = rand_bits(rng, (G, w, D))
    k = rand_bits(rng, (N, D))
    qt = torch.as_tensor(onp.widen(q))
    kt = torch.as_tensor(onp.widen(k))
    allowed = torch.arange(N)[None, :] <= (M + torch.arange(w))[:, None]   # [w, N]
    p = torch.nn.functional.scaled_dot_product_attention(
        qt[None], kt[None, None].expand(1, G, N, D), torch.eye(N, dtype=torch.float64)
        [None, None].expand(1, G, N, N), attn_mask=allowed[None, None])[0]   # [G, w, N]
    a = p.mean(dim=1)[:, :M]
    ihat = a.max(dim=0).values.numpy()
    got = IMPLS[impl].importance(q, k, N)
    np.testing.assert_allclose(got, ihat / ihat.sum(), rtol=1e-10)


# --------------------------------------------------------------------------
# Redundancy
# --------------------------------------------------------------------------

def _orthogonal_case():
    """N=12, w=2, D=16.  Keys are scaled basis vectors; positions 0, 4, 7 share
    direction e0 (scales 1, 2, 0.5); position 10 (window) repeats the
    direction of position 2; position 3 is the zero vector."""
    D, N, w = 16, 12, 2
    rows = []
    for i in range(N):
        if i in (0, 4, 7):
            rows.append(E(0, D, {0: 1.0, 4: 2.0, 7: 0.5}[i]))
        elif i == 10:
            rows.append(E(2, D, 3.0))
        elif i == 3:
            rows.append(np.zeros(D, dtype=np.float32))
        else:
            rows.append(E(i, D, 1.0 + 0.25 * i))
    return bits(rows), N, w


@pytest.mark.parametrize("impl", IMPLS)
def test_redundancy_closed_forms_mean(impl):
    """MEAN: r_i = (#other keys sharing i's direction)/(N-1), zero key -> 0.

    Pins the diagonal exclusion (else every r gets +1/(N-1)), the divisor
    N-1, the window keys counting as "other cached keys", the zero-norm clamp
    (a zero key has similarity 0 with everything) and the normalisation
    (scales 1, 2, 0.5 of the same direction all count as copies).
    """
    k, N, w = _orthogonal_case()
    r = IMPLS[impl].redundancy(k, N, w, oracle.RED_MEAN)
    want = np.zeros(N - w)
    for i in (0, 4, 7):
        want[i] = 2.0 / (N - 1)
    want[2] = 1.0 / (N - 1)
    np.testing.assert_allclose(r, want, atol=1e-15)


@pytest.mark.parametrize("impl", IMPLS)
def test_redundancy_closed_forms_max(impl):
    """MAX: copies (any positive scale) -> 1, orthogonal or zero -> 0."""
    k, N, w = _orthogonal_case()
    r = IMPLS[impl].redundancy(k, N, w, oracle.RED_MAX)
    want = np.zeros(N - w)
    want[[0, 4, 7, 2]] = 1.0
    np.testing.assert_allclose(r, want, atol=1e-15)


@pytest.mark.parametrize("impl", IMPLS)
def test_redundancy_antipodal(impl):
    """A key and its negation have cosine -1: MEAN r = -1/(N-1) for both."""
    D, N, w = 8, 6, 1
    rows = [E(0, D, 1.0), E(0, D, -2.0)] + [E(i, D) for i in range(2, N)]
    r = IMPLS[impl].redundancy(bits(rows), N, w, oracle.RED_MEAN)
    want = np.zeros(N - w)
    want[0] = want[1] = -1.0 / (N - 1)
    np.testing.assert_allclose(r, want, atol=1e-15)


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("mode", [oracle.RED_MEAN, oracle.RED_MAX])
def test_redundancy_scale_invariant(impl, mode):
    """Cosine similarity ignores key length: scaling keys by powers of two
    (exact in bf16) leaves r unchanged."""
    rng = np.random.default_rng(3)
    N, w, D = 64, 8, 128
    k = rand_bits(rng, (N, D))
    kf = onp.widen(k).astype(np.float32)
    scales = (2.0 ** rng.integers(-3, 4, size=N)).astype(np.float32)
    k2 = bits(kf * scales[:, None])
    a = IMPLS[impl].redundancy(k, N, w, mode)
    b = IMPLS[impl].redundancy(k2, N, w, mode)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-15)


def test_redundancy_mean_closed_form_row_sum():
    """MEAN through the row sum of normalised keys equals the masked mean."""
    rng = np.random.default_rng(4)
    N, w, D = 150, 8, 128
    k = rand_bits(rng, (N, D))
    a = oracle.redundancy(k, N, w, oracle.RED_MEAN)
    b = onp.redundancy_mean_closed_form(k, N, w)
    np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-14)


@pytest.mark.parametrize("impl", IMPLS)
def test_exact_duplicates_get_maximal_R_under_max(impl):
    """Two exact copies in a random cache: r = 1 (the largest possible cosine)."""
    rng = np.random.default_rng(5)
    N, w, D = 80, 8, 128
    kf = rng.standard_normal((N, D)).astype(np.float32)
    kf[30] = kf[11]
    k = torch.as_tensor(kf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    r = IMPLS[impl].redundancy(k, N, w, oracle.RED_MAX)
    R = IMPLS[impl].softmax(r)
    assert abs(r[11] - 1.0) < 1e-12 and abs(r[30] - 1.0) < 1e-12
    assert R[11] == R.max() and R[30] == R.max()
    assert np.sort(r)[-3] < 1.0 - 1e-3


# --------------------------------------------------------------------------
# Softmax, joint score, selection
# --------------------------------------------------------------------------

@pytest.mark.parametrize("impl", IMPLS)
def test_softmax_properties(impl):
    np.testing.assert_allclose(IMPLS[impl].softmax(np.zeros(7)), np.full(7, 1 / 7), rtol=1e-15)
    x = np.array([0.0, math.log(2.0), math.log(5.0)])
    np.testing.assert_allclose(IMPLS[impl].softmax(x), np.array([1, 2, 5]) / 8.0, rtol=1e-14)


def _brute_best(Z, kk):
    """Lexicographically smallest index tuple among k-subsets maximising sum Z."""
    best, best_set = None, None
    for s in itertools.combinations(range(len(Z)), kk):
        v = math.fsum(Z[list(s)])
        if best is None or v > best:
            best, best_set = v, s
    return list(best_set)


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("seed", range(6))
def test_select_brute_force(impl, seed):
    """Every k-subset of the candidates: the oracle's choice maximises sum Z."""
    rng = np.random.default_rng(100 + seed)
    N = int(rng.integers(6, 13))
    w = int(rng.integers(1, 4))
    budget = int(rng.integers(w + 1, N))
    G, D = 2, 16
    q = rand_bits(rng, (G, w, D))
    k = rand_bits(rng, (N, D))
    lam = float(rng.choice([0.0, 0.1, 0.5, 1.0]))
    u = IMPLS[impl].unit(q, k, N, budget, lam) if impl == "numpy" else oracle.unit(q, k, N, budget, lam)
    kk = budget - w
    want = _brute_best(u["Z"], kk) + list(range(N - w, N))
    assert list(u["kept"]) == want


@pytest.mark.parametrize("impl", IMPLS)
def test_select_ties_keep_lowest_index(impl):
    """All keys equal: all Z equal, so the lowest indices survive (plus the window)."""
    rng = np.random.default_rng(8)
    N, w, D, budget = 40, 4, 32, 20
    row = rand_bits(rng, (1, D))
    k = np.repeat(row, N, axis=0)
    q = rand_bits(rng, (2, w, D))
    u = IMPLS[impl].unit(q, k, N, budget, 0.1)
    assert np.ptp(u["Z"]) == 0.0
    assert list(u["kept"]) == list(range(budget - w)) + list(range(N - w, N))


@pytest.mark.parametrize("impl", IMPLS)
def test_lambda_one_is_attention_only(impl):
    """lambda = 1: kept candidates are the top-k of I (atlas.scime.ai ablation row)."""
    rng = np.random.default_rng(9)
    N, w, D, budget = 120, 8, 64, 60
    q = rand_bits(rng, (4, w, D))
    k = rand_bits(rng, (N, D))
    u = IMPLS[impl].unit(q, k, N, budget, 1.0)
    M = N - w
    top = np.argsort(-u["I"], kind="stable")[: budget - w]
    assert set(u["kept"][: budget - w]) == set(top.tolist())
    assert list(u["kept"][budget - w:]) == list(range(M, N))


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("mode", [oracle.RED_MEAN, oracle.RED_MAX])
def test_lambda_zero_is_redundancy_only(impl, mode):
    """lambda = 0: the most redundant candidates go (Z = -R, softmax is monotone)."""
    rng = np.random.default_rng(10)
    N, w, D, budget = 120, 8, 64, 60
    q = rand_bits(rng, (4, w, D))
    k = rand_bits(rng, (N, D))
    u = IMPLS[impl].unit(q, k, N, budget, 0.0, red_mode=mode)
    least = np.argsort(u["r"], kind="stable")[: budget - w]
    assert set(u["kept"][: budget - w]) == set(least.tolist())


# --------------------------------------------------------------------------
# Invariants, permutation equivariance, compaction
# --------------------------------------------------------------------------

@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("mode", [oracle.RED_MEAN, oracle.RED_MAX])
def test_invariants(impl, mode):
    rng = np.random.default_rng(11)
    N, w, D, budget, G = 200, 8, 128, 150, 4
    q = rand_bits(rng, (G, w, D))
    k = rand_bits(rng, (N, D))
    u = IMPLS[impl].unit(q, k, N, budget, 0.1, red_mode=mode)
    kept = u["kept"]
    assert len(kept) == budget
    assert np.all(np.diff(kept) > 0)
    assert set(range(N - w, N)) <= set(kept.tolist())
    assert abs(u["I"].sum() - 1) < 1e-12 and abs(u["R"].sum() - 1) < 1e-12
    assert np.all(u["I"] > 0) and np.all(u["R"] > 0)


@pytest.mark.parametrize("impl", IMPLS)
def test_permutation_equivariance(impl):
    """Permuting candidate rows permutes I and r identically and maps kept sets."""
    rng = np.random.default_rng(12)
    N, w, D, budget, G = 90, 8, 64, 50, 4
    M = N - w
    q = rand_bits(rng, (G, w, D))
    k = rand_bits(rng, (N, D))
    perm = np.concatenate([rng.permutation(M), np.arange(M, N)])
    u = IMPLS[impl].unit(q, k, N, budget, 0.1)
    v = IMPLS[impl].unit(q, k[perm], N, budget, 0.1)
    np.testing.assert_allclose(v["I"], u["I"][perm[:M]], rtol=1e-12)
    np.testing.assert_allclose(v["r"], u["r"][perm[:M]], rtol=1e-12, atol=1e-15)
    kept_u = set(u["kept"].tolist())
    kept_v = {int(perm[i]) for i in v["kept"]}
    assert kept_u == kept_v


def test_compaction_is_fancy_index():
    rng = np.random.default_rng(13)
    src = rng.integers(0, 65535, size=(50, 128), dtype=np.uint16)
    kept = np.sort(rng.choice(50, size=30, replace=False)).astype(np.int32)
    np.testing.assert_array_equal(oracle.compact(src, kept), src[kept])
    np.testing.assert_array_equal(onp.compact(src, kept), src[kept])


# --------------------------------------------------------------------------
# The two formulations agree
# --------------------------------------------------------------------------

@pytest.mark.parametrize("mode", [oracle.RED_MEAN, oracle.RED_MAX])
@pytest.mark.parametrize("pool", [oracle.POOL_MAX, oracle.POOL_MEAN])
def test_c_and_numpy_twins_agree(mode, pool):
    rng = np.random.default_rng(14)
    for N, w, G, budget in [(160, 8, 4, 120), (257, 8, 5, 200), (33, 3, 2, 20)]:
        q = rand_bits(rng, (G, w, 128))
        k = rand_bits(rng, (N, 128))
        a = oracle.unit(q, k, N, budget, 0.1, red_mode=mode, pool=pool)
        b = onp.unit(q, k, N, budget, 0.1, red_mode=mode, pool=pool)
        for name in ("I", "r", "R", "Z"):
            np.testing.assert_allclose(a[name], b[name], rtol=1e-12, atol=1e-15)
        np.testing.assert_array_equal(a["kept"], b["kept"])


def test_batched_oracle_matches_single_units():
    rng = np.random.default_rng(15)
    U, G, w, D, cap = 5, 4, 8, 128, 100
    q = rand_bits(rng, (U, G, w, D))
    k = rand_bits(rng, (U, cap, D))
    N = np.array([100, 90, 64, 100, 77], dtype=np.int32)
    budget = np.array([60, 50, 40, 80, 30], dtype=np.int32)
    lam = np.array([0.1, 0.0, 1.0, 0.5, 0.1])
    out = oracle.units(q, k, N, budget, lam, n_threads=2)
    for u in range(U):
        one = oracle.unit(q[u], k[u], int(N[u]), int(budget[u]), float(lam[u]))
        M = int(N[u]) - w
        for name in ("I", "r", "R", "Z"):
            np.testing.assert_array_equal(out[name][u, :M], one[name])
        np.testing.assert_array_equal(out["kept"][u, : budget[u]], one["kept"])
