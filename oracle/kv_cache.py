"""Paged KV cache write side, plain numpy (TEST INFRASTRUCTURE ONLY).

Source: "Recomendador generativo HSTU com Dynamo-Triton" (KV cache section):
the attention state of a user's stable prefix is kept in a paged GPU table;
a request computes only its new actions and candidates, and afterwards the
new actions are appended to the table (candidates are not cached).  The pages
describe no allocator, so the policy below is the library's own, stated as
its definition:
  * free pages form a stack free_pages[0 : free_count]; the top is the end;
  * append: users in order take the pages they need from the top, user u's
    j-th new page being free_pages[free_count - 1 - (pages taken by users
    before u) - j]; token j of the append lands at position cached_len + j,
    i.e. page  table[u][(cached_len + j) // P], slot (cached_len + j) % P;
  * evict: users in order push their pages (page-table order) on the stack,
    their table row becomes -1 and their cached length 0;
  * a call that does not fit (stack too small, a table row too short) or that
    meets a bad length or page id changes nothing and reports its status.
Every function returns new arrays; the inputs are not modified.
"""
from __future__ import annotations

import numpy as np

OK, ERR_LENGTH, ERR_PAGE, ERR_POOL = 0, -4, -9, -10


def _pages(n: int, P: int) -> int:
    return -(-n // P)


def kv_append(k_pool, v_pool, page_table, cached_lens, free_pages, free_count, k_new, v_new, new_offsets,
              num_append=None):
    """Returns (status, k_pool, v_pool, page_table, cached_lens, free_pages, free_count).

    k_pool, v_pool: [num_pages, H, P, d]; k_new, v_new: [T_new, H, d]."""
    k_pool, v_pool = np.array(k_pool, copy=True), np.array(v_pool, copy=True)
    table = np.array(page_table, dtype=np.int64, copy=True)
    lens = np.array(cached_lens, dtype=np.int64, copy=True)
    free = np.array(free_pages, dtype=np.int64, copy=True)
    fc = int(free_count)
    num_pages, H, P, d = k_pool.shape
    B, max_pages = table.shape
    off = np.asarray(new_offsets, dtype=np.int64)
    unchanged = (OK, k_pool, v_pool, table, lens, free, fc)
    apps, needs = [], []
    status = OK
    for u in range(B):
        L, n_new = int(lens[u]), int(off[u + 1] - off[u])
        app = n_new if num_append is None else int(num_append[u])
        if L < 0 or off[u] < 0 or off[u + 1] > len(k_new) or n_new < 0 or app < 0 or app > n_new:
            return (ERR_LENGTH,) + unchanged[1:]
        if _pages(L + app, P) > max_pages:
            status = status or ERR_POOL
            apps.append(0)
            needs.append(0)
            continue
        if app > 0 and L % P != 0 and not (0 <= table[u, L // P] < num_pages):
            status = status or ERR_PAGE
        apps.append(app)
        needs.append(_pages(L + app, P) - _pages(L, P))
    total = sum(needs)
    if status == OK and (total > fc or fc > num_pages):
        status = ERR_POOL
    if status == OK and any(not (0 <= free[x] < num_pages) for x in range(fc - total, fc)):
        status = ERR_PAGE
    if status != OK:
        return (status,) + unchanged[1:]
    taken = 0
    for u in range(B):
        L, app = int(lens[u]), apps[u]
        have = _pages(L, P)
        for j in range(needs[u]):
            table[u, have + j] = free[fc - 1 - taken - j]
        taken += needs[u]
        for j in range(app):
            pos = L + j
            page, slot = table[u, pos // P], pos % P
            k_pool[page, :, slot, :] = k_new[off[u] + j]
            v_pool[page, :, slot, :] = v_new[off[u] + j]
        lens[u] = L + app
    return OK, k_pool, v_pool, table, lens, free, fc - total


def kv_evict(page_table, cached_lens, free_pages, free_count, evict_mask, page_size: int, num_pages: int):
    """Returns (status, page_table, cached_lens, free_pages, free_count)."""
    table = np.array(page_table, dtype=np.int64, copy=True)
    lens = np.array(cached_lens, dtype=np.int64, copy=True)
    free = np.array(free_pages, dtype=np.int64, copy=True)
    fc = int(free_count)
    B, max_pages = table.shape
    unchanged = (OK, table, lens, free, fc)
    counts = []
    for u in range(B):
        if not evict_mask[u]:
            counts.append(0)
            continue
        L = int(lens[u])
        if L < 0 or _pages(L, page_size) > max_pages:
            return (ERR_LENGTH,) + unchanged[1:]
        cnt = _pages(L, page_size)
        if any(not (0 <= table[u, j] < num_pages) for j in range(cnt)):
            return (ERR_PAGE,) + unchanged[1:]
        counts.append(cnt)
    if fc < 0 or fc + sum(counts) > num_pages:
        return (ERR_POOL,) + unchanged[1:]
    for u in range(B):
        for j in range(counts[u]):
            free[fc + j] = table[u, j]
            table[u, j] = -1
        fc += counts[u]
        if evict_mask[u]:
            lens[u] = 0
    return OK, table, lens, free, fc


def gather_prefix(k_pool, page_table, cached_lens, u: int):
    """The cached K (or V) of user u as [L, H, d], read through the table."""
    num_pages, H, P, d = k_pool.shape
    L = int(cached_lens[u])
    out = np.empty((L, H, d), dtype=np.asarray(k_pool).dtype)
    for pos in range(L):
        out[pos] = np.asarray(k_pool)[page_table[u][pos // P], :, pos % P, :]
    return out
