"""Pins of the paged-cache definitions (page-table gather, freed pages)."""
import numpy as np

from oracle import rkv_oracle_np as onp


def test_identity_table_is_the_contiguous_cache():
    g = np.random.default_rng(0)
    H, P, npages, D = 3, 16, 5, 8
    pool = g.integers(0, 65535, size=(npages, H, P, D)).astype(np.uint16)
    # one sequence owning pages 0..4 in order: logical row i = page i // P, slot i % P
    for h in range(H):
        rows = onp.paged_rows(pool, np.arange(npages), h, npages * P, P)
        np.testing.assert_array_equal(rows, pool[:, h].reshape(npages * P, D))


def test_permuted_table_by_hand():
    P, D = 4, 2
    pool = np.arange(6 * 1 * P * D, dtype=np.uint16).reshape(6, 1, P, D)
    bt = [5, 2, 0]
    rows = onp.paged_rows(pool, bt, 0, 10, P)
    assert rows[0].tolist() == pool[5, 0, 0].tolist()
    assert rows[5].tolist() == pool[2, 0, 1].tolist()      # row 5 = page bt[1], slot 1
    assert rows[9].tolist() == pool[0, 0, 1].tolist()      # row 9 = page bt[2], slot 1


def test_freed_pages():
    bt = [7, 3, 9, 1, 4]
    assert onp.freed_pages(bt, 40, 24, 16) == [9]            # 3 pages in use, 2 needed
    assert onp.freed_pages(bt, 80, 16, 16) == [3, 9, 1, 4]
    assert onp.freed_pages(bt, 40, 33, 16) == []             # still 3 pages
    bt9 = list(range(100, 109))
    assert onp.freed_pages(bt9, 1152, 1024, 128) == [108]
    for P in (16, 32, 64, 128):
        for N, b in ((1152, 1024), (1766, 1638), (300, 100)):
            n = len(onp.freed_pages(list(range(200)), N, b, P))
            assert n == -(-N // P) - -(-b // P)
