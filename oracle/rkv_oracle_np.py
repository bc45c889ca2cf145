"""NumPy float64 twin of the C oracle of the R-KV compression step.

TEST INFRASTRUCTURE ONLY: only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module.  It shares no code with the CUDA path
and none with ``rkv_oracle.c`` either: it is a second, vectorised formulation
of the same definition, used to cross-check the C loops.

Per unit (one sequence, layer and KV head), with N cached tokens, window w,
M = N - w candidates and k = budget - w kept candidates:

* importance: scaled-softmax attention of the last w queries of every query
  head in the GQA group (query j at position M+j sees keys 0..M+j), mean over
  the w queries, max over the group, renormalised over the candidates
  (R-KV pages: sourcepulse "How It Works" -- importance from attention
  weights; atlas.scime.ai "Measured effects" -- max pooling over GQA heads);
* redundancy: cosine similarity of L2-normalised keys, mean (or max) over the
  other N-1 cached keys, then softmax over the candidates (atlas.scime.ai
  summary and "Approach" -- key-vector cosine similarity);
* joint score Z = lambda I - (1 - lambda) R (atlas.scime.ai "Approach");
* keep the top k by (Z desc, index asc) plus the window, ascending
  (sourcepulse "How It Works"; hysenlabs decode-time section on window_size);
* compaction: gather the kept rows of K and V.
"""
from __future__ import annotations

import numpy as np

POOL_MAX, POOL_MEAN = 0, 1
RED_MEAN, RED_MAX = 0, 1


def widen(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64 values."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def importance(q_bits, k_bits, N, pool=POOL_MAX):
    """q_bits: [G, w, D], k_bits: [>=N, D] -> I: [M] (sums to 1)."""
    q = widen(q_bits)
    k = widen(k_bits)[:N]
    G, w, D = q.shape
    M = N - w
    logits = np.einsum("gjd,nd->gjn", q, k) / np.sqrt(D)
    pos = M + np.arange(w)                       # position of query j
    visible = np.arange(N)[None, :] <= pos[:, None]   # [w, N]
    logits = np.where(visible[None], logits, -np.inf)
    logits = logits - logits.max(axis=2, keepdims=True)
    p = np.exp(logits)
    p = p / p.sum(axis=2, keepdims=True)
    a = p.mean(axis=1)[:, :M]                    # [G, M]: window mean
    ihat = a.max(axis=0) if pool == POOL_MAX else a.mean(axis=0)
    return ihat / ihat.sum()


def inv_norm(k_bits, N):
    k = widen(k_bits)[:N]
    return 1.0 / np.maximum(np.sqrt((k * k).sum(axis=1)), 1e-12)


def redundancy(k_bits, N, w, mode=RED_MEAN):
    """Raw redundancy r: [M] from the masked cosine-similarity matrix."""
    k = widen(k_bits)[:N]
    M = N - w
    kh = k * inv_norm(k_bits, N)[:, None]
    C = kh @ kh.T
    off = ~np.eye(N, dtype=bool)
    if mode == RED_MAX:
        return np.where(off, C, -np.inf)[:M].max(axis=1)
    return np.where(off, C, 0.0)[:M].sum(axis=1) / (N - 1)


def redundancy_mean_closed_form(k_bits, N, w):
    """MEAN redundancy through the row sum: r_i = (khat_i . S - khat_i . khat_i)/(N-1)."""
    k = widen(k_bits)[:N]
    M = N - w
    kh = k * inv_norm(k_bits, N)[:, None]
    S = kh.sum(axis=0)
    return ((kh[:M] @ S) - (kh[:M] * kh[:M]).sum(axis=1)) / (N - 1)


def softmax(x):
    e = np.exp(x - np.max(x))
    return e / e.sum()


def joint(I, R, lam):
    return lam * I - (1.0 - lam) * R


def select(Z, N, budget):
    """kept: [budget] int32, ascending; candidates by (Z desc, index asc) then window."""
    M = Z.shape[0]
    w = N - M
    kk = budget - w
    order = np.lexsort((np.arange(M), -Z))       # primary -Z, secondary index
    chosen = np.sort(order[:kk])
    return np.concatenate([chosen, np.arange(M, N)]).astype(np.int32)


def compact(src_bits, kept):
    return np.asarray(src_bits)[np.asarray(kept)]


def shared_select(Z_heads, N, budget):
    """One kept set for all heads of a (sequence, layer): the heads' joint scores
    summed (the tensor-parallel ranks' all-reduce), then the per-head rule."""
    Zsum = np.asarray(Z_heads, dtype=np.float64).sum(axis=0)
    return Zsum, select(Zsum, N, budget)


def unit(q_bits, k_bits, N, budget, lam, red_mode=RED_MEAN, pool=POOL_MAX):
    """Whole step for one unit; returns dict of I, r, R, Z (float64 [M]) and kept."""
    w = q_bits.shape[1]
    I = importance(q_bits, k_bits, N, pool)
    r = redundancy(k_bits, N, w, red_mode)
    R = softmax(r)
    Z = joint(I, R, lam)
    kept = select(Z, N, budget)
    return {"I": I, "r": r, "R": R, "Z": Z, "kept": kept}


# ---------------------------------------------------------------- paged caches
# A paged cache keeps each layer's keys (and values) in a pool of fixed-size
# pages, pool[page, head, slot, :], and each sequence owns a list of pages
# (its block table): logical row i of a sequence lives in page
# block_table[i // P] at slot i % P.  Compressing a sequence to `budget` rows
# leaves its pages ceil(budget / P) .. ceil(N / P) - 1 empty, and they go back
# to the allocator -- the FREE_BLOCKS return path of the vLLM port (hysenlabs
# write-up, decode-time section: physical eviction returns freed blocks).

def paged_rows(pool_bits, block_table_row, h, n_rows, page_rows):
    """Logical rows 0..n_rows-1 of KV head h, gathered through the block table."""
    pool = np.asarray(pool_bits)
    bt = np.asarray(block_table_row)
    return np.stack([pool[bt[i // page_rows], h, i % page_rows] for i in range(n_rows)])


def freed_pages(block_table_row, n_tokens, budget, page_rows):
    """Pages a sequence no longer needs after compaction from n_tokens to budget rows."""
    keep = -(-budget // page_rows)
    used = -(-n_tokens // page_rows)
    return [int(x) for x in np.asarray(block_table_row)[keep:used]]
