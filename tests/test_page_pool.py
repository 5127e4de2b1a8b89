"""The host-side page pool (pmla_page_pool_*): no page is handed out twice,
frees are reusable, every call is all-or-nothing.  CPU only."""
import numpy as np
import pytest

import paged_mla_attention_b200 as pm


def test_alloc_all_then_exhausted():
    pool = pm.PagePool(10)
    a = pool.alloc(10)
    assert sorted(a.tolist()) == list(range(10)) and pool.num_free == 0
    with pytest.raises(pm.PmlaError):
        pool.alloc(1)
    assert pool.num_free == 0


def test_exhaustion_allocates_nothing():
    pool = pm.PagePool(8)
    pool.alloc(5)
    with pytest.raises(pm.PmlaError):
        pool.alloc(4)            # only 3 left
    assert pool.num_free == 3
    assert len(pool.alloc(3)) == 3


def test_free_then_reuse():
    pool = pm.PagePool(6)
    a = pool.alloc(6)
    pool.free(a[:2])
    assert pool.num_free == 2
    b = pool.alloc(2)
    assert sorted(b.tolist()) == sorted(a[:2].tolist())


@pytest.mark.parametrize("bad", [[7], [-1], [100], [1, 1]])
def test_bad_frees_change_nothing(bad):
    pool = pm.PagePool(8)
    a = pool.alloc(4)            # ids 0..3 allocated, 4..7 free
    before = pool.num_free
    with pytest.raises(pm.PmlaError):
        pool.free(bad if bad != [1, 1] else [a[1], a[1]])
    assert pool.num_free == before
    pool.free(a)                 # the real ones still free fine
    assert pool.num_free == 8


def test_double_free_rejected():
    pool = pm.PagePool(4)
    a = pool.alloc(2)
    pool.free(a)
    with pytest.raises(pm.PmlaError):
        pool.free(a)
    assert pool.num_free == 4


def test_grow_and_release_sequence_rows():
    pool = pm.PagePool(20)
    row = np.full(8, -1, dtype=np.int32)
    pool.grow(row, 0, 1)                     # 1 token -> 1 page
    assert row[0] >= 0 and np.all(row[1:] == -1)
    pool.grow(row, 1, 64)                    # still one page
    assert np.all(row[1:] == -1)
    pool.grow(row, 64, 65)                   # second page
    assert row[1] >= 0 and row[1] != row[0]
    pool.grow(row, 65, 300)                  # pages 2..4
    assert np.all(row[:5] >= 0) and np.all(row[5:] == -1) and len(set(row[:5].tolist())) == 5
    with pytest.raises(pm.PmlaError):
        pool.grow(row, 300, 8 * 64 + 1)      # past the row
    assert pool.num_free == 15
    pool.release(row, 300)
    assert pool.num_free == 20


def test_random_churn_keeps_pages_disjoint():
    rng = np.random.default_rng(0)
    pool = pm.PagePool(500)
    rows = {s: (np.full(40, -1, dtype=np.int32), 0) for s in range(12)}
    for step in range(3000):
        s = int(rng.integers(12))
        row, L = rows[s]
        if rng.random() < 0.15 and L > 0:
            pool.release(row, L)
            rows[s] = (np.full(40, -1, dtype=np.int32), 0)
            continue
        new_len = min(L + int(rng.integers(1, 200)), 40 * 64)
        try:
            pool.grow(row, L, new_len)
            rows[s] = (row, new_len)
        except pm.PmlaError:
            pass                               # exhausted: the row is unchanged
        used = [r[:(l + 63) // 64] for r, l in rows.values()]
        flat = np.concatenate(used) if used else np.array([], dtype=np.int32)
        assert len(set(flat.tolist())) == len(flat), "a page is owned by two sequences"
        assert pool.num_free + len(flat) == 500
