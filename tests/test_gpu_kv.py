"""GPU tests of the paged KV cache write side: append/evict bit-exact against
the oracle's allocator model, all-or-nothing failures, and append-then-attend
equal to a full recompute over the unpaged sequence."""
import numpy as np
import pytest
import torch

import generative_recommender_attention_jagged_b200 as hstu
import oracle
import synth
from oracle import kv_cache as okv

from .gpu_helpers import BF16_TOL, dev, host64, rel_err

pytestmark = pytest.mark.gpu

H, D = 4, 128


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy() if t.dtype == torch.bfloat16 else t.detach().cpu().numpy()


class Cache:
    """Device cache state plus the oracle's copy of it."""

    def __init__(self, B, num_pages, max_pages, P, seed):
        rng = np.random.default_rng(seed)
        self.P, self.num_pages = P, num_pages
        pool = synth.draw_normal(rng, (num_pages, H, P, D), 1.0, torch.bfloat16)
        self.k_pool, self.v_pool = pool.clone().cuda(), (pool * 2).cuda()
        self.table = torch.full((B, max_pages), -1, dtype=torch.int32, device="cuda")
        self.lens = torch.zeros(B, dtype=torch.int32, device="cuda")
        self.free = torch.from_numpy(rng.permutation(num_pages).astype(np.int32)).cuda()
        self.fc = torch.tensor([num_pages], dtype=torch.int32, device="cuda")
        # oracle state: bf16 bit patterns as int16 arrays
        self.o = [bits(self.k_pool), bits(self.v_pool), self.table.cpu().numpy(), self.lens.cpu().numpy(),
                  self.free.cpu().numpy(), num_pages]

    def append(self, counts, num_append=None, seed=0):
        rng = np.random.default_rng(seed)
        T = int(sum(counts))
        k = synth.draw_normal(rng, (T, H, D), 1.0, torch.bfloat16)
        v = synth.draw_normal(rng, (T, H, D), 1.0, torch.bfloat16)
        off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        ws = hstu.hstu_kv_append(k.cuda(), v.cuda(), dev(off), self.k_pool, self.v_pool, self.table, self.lens,
                                 self.free, self.fc, num_append=dev(num_append, torch.int32))
        status = hstu.hstu_check_device_error(ws)
        st, *rest = okv.kv_append(self.o[0], self.o[1], self.o[2], self.o[3], self.o[4], self.o[5],
                                  bits(k), bits(v), off, num_append)
        if st == okv.OK:
            self.o = rest
        return status, st, k, v, off

    def evict(self, mask):
        ws = hstu.hstu_kv_evict(dev(np.asarray(mask, np.int32)), self.k_pool, self.table, self.lens, self.free,
                                self.fc)
        status = hstu.hstu_check_device_error(ws)
        st, table, lens, free, fc = okv.kv_evict(self.o[2], self.o[3], self.o[4], self.o[5], mask, self.P,
                                                 self.num_pages)
        if st == okv.OK:
            self.o = [self.o[0], self.o[1], table, lens, free, fc]
        return status, st

    def assert_matches_oracle(self):
        k_o, v_o, table, lens, free, fc = self.o
        assert int(self.fc.item()) == fc
        assert np.array_equal(self.table.cpu().numpy(), table)
        assert np.array_equal(self.lens.cpu().numpy(), lens)
        assert np.array_equal(self.free.cpu().numpy()[:fc], free[:fc])
        assert np.array_equal(bits(self.k_pool), k_o)
        assert np.array_equal(bits(self.v_pool), v_o)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_append_evict_sequences_bit_exact(seed):
    rng = np.random.default_rng(500 + seed)
    B, P = 5, 32
    c = Cache(B, num_pages=60, max_pages=12, P=P, seed=seed)
    for step in range(10):
        if rng.random() < 0.3:
            status, st = c.evict((rng.random(B) < 0.4).astype(np.int32))
            assert status == st == 0
        else:
            counts = rng.integers(0, 70, size=B)
            acts = np.minimum(counts, rng.integers(0, 70, size=B)).astype(np.int32)
            status, st, *_ = c.append(counts, acts if step % 2 else None, seed=1000 * seed + step)
            assert status == st                       # 0, or -10 when the pool / a row is full
        c.assert_matches_oracle()


def test_pool_exhausted_is_reported_and_changes_nothing():
    c = Cache(3, num_pages=5, max_pages=8, P=32, seed=9)
    status, st, *_ = c.append([100, 90, 10], seed=1)   # 4 + 3 + 1 pages > 5
    assert status == st == okv.ERR_POOL == -10
    c.assert_matches_oracle()                            # oracle state was not advanced either
    status, st, *_ = c.append([40, 30, 10], seed=2)      # 2 + 1 + 1 pages: fits
    assert status == st == 0
    c.assert_matches_oracle()


def test_bad_page_id_in_a_partial_page_is_reported():
    c = Cache(2, num_pages=8, max_pages=4, P=32, seed=3)
    assert c.append([10, 0], seed=4)[0] == 0
    c.table[0, 0] = 99                                   # corrupt the partly filled page of user 0
    c.o[2][0, 0] = 99
    status, st, *_ = c.append([5, 0], seed=5)
    assert status == st == -9
    c.assert_matches_oracle()


def test_append_then_attend_equals_full_recompute():
    """Request 1 appends its actions to the cache; request 2 is answered by the
    paged path over the updated cache and must equal attention over the whole
    unpaged sequence (prefix + request-1 actions + request-2 tokens)."""
    rng = np.random.default_rng(77)
    cached = [100, 37, 64]
    pb = synth.paged_batch(cached, 10, 5, H, D, 512, rng=rng, spare_pages=12, poison=True)
    B, P = len(cached), pb.page_size
    num_pages = pb.k_pool.shape[0]
    used = set(int(x) for x in pb.kv_page_table.ravel() if x >= 0)
    free = np.array([p for p in range(num_pages) if p not in used], np.int32)
    # the page table needs room for the appended pages
    table = np.full((B, pb.kv_page_table.shape[1] + 2), -1, np.int32)
    table[:, :pb.kv_page_table.shape[1]] = pb.kv_page_table
    k_pool, v_pool = dev(pb.k_pool), dev(pb.v_pool)
    d_table, d_lens = dev(table), dev(pb.cached_lens, torch.int32)
    d_free, d_fc = dev(free), torch.tensor([len(free)], dtype=torch.int32, device="cuda")
    # request 1: cache its 10 actions (not the 5 candidates)
    ws = hstu.hstu_kv_append(dev(pb.k), dev(pb.v), dev(pb.new_offsets, torch.int32), k_pool, v_pool, d_table,
                             d_lens, d_free, d_fc, num_append=dev(np.full(B, 10, np.int32)))
    assert hstu.hstu_check_device_error(ws) == 0
    assert d_lens.cpu().tolist() == [c + 10 for c in cached]
    # request 2: 7 actions + 3 candidates per user, after the cached history
    n_act, n_cand = 7, 3
    T2 = B * (n_act + n_cand)
    q2, k2, v2 = (synth.draw_normal(rng, (T2, H, D), 1.0, torch.bfloat16) for _ in range(3))
    u2 = synth.draw_normal(rng, (T2, H * D), 1.0, torch.bfloat16)
    off2 = np.arange(0, T2 + 1, n_act + n_cand, dtype=np.int32)
    ts_full, seq_len = [], []
    for b in range(B):
        L = cached[b] + 10
        t_hist = pb.timestamps[pb.ts_offsets[b]:pb.ts_offsets[b] + L]
        gaps = rng.integers(1, 900, size=n_act)
        t_act = t_hist[-1] + np.cumsum(gaps)
        ts_full.append(np.concatenate([t_hist, t_act, np.full(n_cand, t_act[-1])]))
        seq_len.append(L + n_act + n_cand)
    ts_full_cat = np.concatenate(ts_full).astype(np.int64)
    ts_off = np.concatenate([[0], np.cumsum(seq_len)]).astype(np.int32)
    y = hstu.hstu_attn_fwd_paged(q2.cuda(), k2.cuda(), v2.cuda(), u2.cuda(), dev(off2), dev(ts_full_cat),
                                 dev(ts_off), dev(pb.rab_pos, torch.float32), dev(pb.rab_ts, torch.float32),
                                 k_pool, v_pool, d_table, d_lens, n_max=pb.n_max,
                                 num_candidates=dev(np.full(B, n_cand, np.int32)))
    torch.cuda.synchronize()
    # full recompute: every user's whole sequence, unpaged
    qs, ks, vs, us, rows = [], [], [], [], []
    base = 0
    for b in range(B):
        L0 = cached[b]
        a0, a1 = int(pb.new_offsets[b]), int(pb.new_offsets[b]) + 10
        r0, r1 = int(off2[b]), int(off2[b + 1])
        ks.append(torch.cat([pb.k_prefix[b], pb.k[a0:a1], k2[r0:r1]]))
        vs.append(torch.cat([pb.v_prefix[b], pb.v[a0:a1], v2[r0:r1]]))
        n_old = L0 + 10
        qs.append(torch.cat([torch.zeros(n_old, H, D, dtype=torch.bfloat16), q2[r0:r1]]))
        us.append(torch.cat([torch.zeros(n_old, H * D, dtype=torch.bfloat16), u2[r0:r1]]))
        rows += list(range(base + n_old, base + seq_len[b]))
        base += seq_len[b]
    want = oracle.attn_jagged(torch.cat(qs), torch.cat(ks), torch.cat(vs), torch.cat(us), ts_off, ts_full_cat,
                              np.full(B, n_cand, np.int32), pb.rab_pos, pb.rab_ts, pb.alpha, pb.n_max,
                              rows=np.array(rows))
    assert rel_err(host64(y), want) <= BF16_TOL
