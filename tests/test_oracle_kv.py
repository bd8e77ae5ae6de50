"""Pins of the KV-cache write-side oracle (oracle/kv_cache.py) against what a
paged cache must do, independent of the allocator's own code: appended tokens
read back through the page table in order, pages are conserved, the policy's
stack order holds on hand-worked cases, and calls that do not fit change
nothing."""
import numpy as np
import pytest

from oracle import kv_cache as kv

H, D, P = 2, 4, 4


def empty_cache(B=3, num_pages=10, max_pages=4):
    k_pool = np.full((num_pages, H, P, D), -1.0)
    v_pool = np.full((num_pages, H, P, D), -2.0)
    table = np.full((B, max_pages), -1, dtype=np.int64)
    lens = np.zeros(B, dtype=np.int64)
    free = np.arange(num_pages, dtype=np.int64)   # top of the stack = the last entry
    return k_pool, v_pool, table, lens, free, num_pages


def tokens(counts, seed):
    rng = np.random.default_rng(seed)
    T = int(sum(counts))
    k = rng.integers(0, 1000, size=(T, H, D)).astype(np.float64)
    v = rng.integers(0, 1000, size=(T, H, D)).astype(np.float64)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    return k, v, off


def test_hand_worked_first_append():
    k_pool, v_pool, table, lens, free, fc = empty_cache()
    k, v, off = tokens([5, 0, 4], 1)
    st, k_pool, v_pool, table, lens, free, fc = kv.kv_append(k_pool, v_pool, table, lens, free, fc, k, v, off)
    assert st == kv.OK
    # user 0 needs 2 pages: 9 then 8 (top of the stack first); user 1 none; user 2 one page: 7
    assert table[0].tolist() == [9, 8, -1, -1]
    assert table[1].tolist() == [-1, -1, -1, -1]
    assert table[2].tolist() == [7, -1, -1, -1]
    assert lens.tolist() == [5, 0, 4] and fc == 7
    # token 4 of user 0 is slot 0 of its second page
    assert np.array_equal(k_pool[8, :, 0, :], k[4]) and np.array_equal(v_pool[9, :, 3, :], v[3])
    # untouched slots keep their old contents
    assert np.all(k_pool[8, :, 1:, :] == -1.0)


def test_append_fills_the_partial_page_first():
    k_pool, v_pool, table, lens, free, fc = empty_cache()
    k1, v1, off1 = tokens([3, 0, 0], 2)
    _, k_pool, v_pool, table, lens, free, fc = kv.kv_append(k_pool, v_pool, table, lens, free, fc, k1, v1, off1)
    k2, v2, off2 = tokens([2, 0, 0], 3)
    st, k_pool, v_pool, table, lens, free, fc = kv.kv_append(k_pool, v_pool, table, lens, free, fc, k2, v2, off2)
    assert st == kv.OK
    assert table[0].tolist() == [9, 8, -1, -1] and lens[0] == 5 and fc == 8
    assert np.array_equal(k_pool[9, :, 3, :], k2[0]) and np.array_equal(k_pool[8, :, 0, :], k2[1])


def test_num_append_caches_only_the_actions():
    k_pool, v_pool, table, lens, free, fc = empty_cache()
    k, v, off = tokens([6, 3, 2], 4)                  # 4 + 2 candidates, 3 + 0, 1 + 1
    st, k_pool, _, table, lens, _, fc = kv.kv_append(k_pool, v_pool, table, lens, free, fc, k, v, off,
                                                     num_append=[4, 3, 1])
    assert st == kv.OK and lens.tolist() == [4, 3, 1]
    got = kv.gather_prefix(k_pool, table, lens, 1)
    assert np.array_equal(got, k[6:9])


@pytest.mark.parametrize("seed", range(6))
def test_random_sequences_read_back_and_conserve_pages(seed):
    rng = np.random.default_rng(100 + seed)
    B, num_pages, max_pages = 4, 24, 8
    k_pool, v_pool, table, lens, free, fc = empty_cache(B, num_pages, max_pages)
    history = [[] for _ in range(B)]                  # what each user's cache must read back as
    for step in range(8):
        if rng.random() < 0.25:
            mask = rng.random(B) < 0.4
            st, table, lens, free, fc = kv.kv_evict(table, lens, free, fc, mask, P, num_pages)
            assert st == kv.OK
            for u in range(B):
                if mask[u]:
                    history[u] = []
            continue
        counts = rng.integers(0, 7, size=B)
        k, v, off = tokens(counts, 1000 * seed + step)
        st, k_pool2, v_pool2, table2, lens2, free2, fc2 = kv.kv_append(k_pool, v_pool, table, lens, free, fc,
                                                                       k, v, off)
        if st == kv.OK:
            k_pool, v_pool, table, lens, free, fc = k_pool2, v_pool2, table2, lens2, free2, fc2
            for u in range(B):
                history[u] += [k[off[u] + j] for j in range(counts[u])]
        else:                                          # did not fit: nothing changed
            assert st == kv.ERR_POOL
            assert np.array_equal(table2, table) and np.array_equal(lens2, lens) and fc2 == fc
        for u in range(B):
            got = kv.gather_prefix(k_pool, table, lens, u)
            want = np.array(history[u]).reshape(-1, H, D)
            assert np.array_equal(got, want)
        # conservation: free pages and mapped pages partition the pool
        mapped = [int(table[u, j]) for u in range(B) for j in range(-(-int(lens[u]) // P))]
        assert sorted(mapped + [int(x) for x in free[:fc]]) == list(range(num_pages))


def test_pool_too_small_changes_nothing():
    k_pool, v_pool, table, lens, free, fc = empty_cache(B=2, num_pages=3, max_pages=4)
    k, v, off = tokens([8, 5], 5)                     # 2 + 2 pages > 3
    st, k2, _, t2, l2, f2, fc2 = kv.kv_append(k_pool, v_pool, table, lens, free, fc, k, v, off)
    assert st == kv.ERR_POOL
    assert np.array_equal(k2, k_pool) and np.array_equal(t2, table) and np.array_equal(l2, lens) and fc2 == fc


def test_row_too_short_changes_nothing():
    k_pool, v_pool, table, lens, free, fc = empty_cache(B=2, num_pages=10, max_pages=2)
    k, v, off = tokens([9, 1], 6)                     # 3 pages > 2 columns
    st = kv.kv_append(k_pool, v_pool, table, lens, free, fc, k, v, off)[0]
    assert st == kv.ERR_POOL


def test_evict_then_append_reuses_pages_lifo():
    k_pool, v_pool, table, lens, free, fc = empty_cache()
    k, v, off = tokens([5, 2, 0], 7)
    _, k_pool, v_pool, table, lens, free, fc = kv.kv_append(k_pool, v_pool, table, lens, free, fc, k, v, off)
    # user 0 holds [9, 8], user 1 holds [7]
    st, table, lens, free, fc = kv.kv_evict(table, lens, free, fc, [1, 0, 0], P, 10)
    assert st == kv.OK and fc == 9 and free[7:9].tolist() == [9, 8] and table[0].tolist() == [-1] * 4
    k2, v2, off2 = tokens([0, 0, 3], 8)
    _, _, _, table, lens, free, fc = kv.kv_append(k_pool, v_pool, table, lens, free, fc, k2, v2, off2)
    assert table[2, 0] == 8 and fc == 8                # the last page pushed is taken first
