"""Pins of the fp64 CPU oracle against things other than itself.

* the time bucket against an exact 60-digit decimal evaluation;
* closed forms (zero scores, constant bias prefix sums, single-token users);
* one-hot bias probes: since SiLU(0) = 0, a bias table that is zero except at
  one entry selects exactly the key pairs that index that entry, which pins
  the relative-position sign and offset, the candidate positions, the mask and
  the time-bucket lookup;
* LayerNorm against torch.nn.functional.layer_norm (a library routine);
* brute force on tiny inputs from explicitly enumerated pair sets;
* invariants: causality, jagged batch = per-user runs, candidate permutation
  equivariance, paged incremental = full recompute, head independence.

Every case is small: the whole file runs in seconds on a CPU.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import layer as olayer
import synth
from tests import exact_bucket as eb


def silu(x):
    return x / (1.0 + math.exp(-x))


# ----------------------------------------------------------------------------
# time bucket
# ----------------------------------------------------------------------------

def test_bucket_edges_are_far_from_integers():
    # the exactness argument of the oracle and of the CUDA threshold table
    assert eb.min_edge_gap() > 1e-3


def test_bucket_at_every_threshold():
    thr = eb.integer_thresholds()
    xs = sorted({max(1, t + dlt) for t in thr for dlt in range(-2, 3)})
    dts = np.array([x - 1 for x in xs if x - 1 < 2**63], dtype=np.int64)
    got = oracle.ts_bucket(dts)
    want = np.array([eb.bucket(int(d)) for d in dts])
    np.testing.assert_array_equal(got, want)
    # threshold table and the direct decimal floor agree
    assert all(eb.bucket(int(d)) == eb.bucket_direct(int(d)) for d in dts[::7])


def test_bucket_special_values():
    dts = np.array([0, 1, -1, 2**62, 2**63 - 1, -(2**63), -(2**63) + 1], dtype=np.int64)
    got = oracle.ts_bucket(dts)
    assert got[0] == 0
    assert got[1] == eb.bucket(1) == 2          # ln 2 / 0.301 = 2.30
    assert got[2] == got[1]                      # |dt|
    assert list(got[3:]) == [127, 127, 127, 127]
    # bucket 127 needs |dt| + 1 >= e^(38.227) ~ 4.0e16
    edge = eb.integer_thresholds()[127]
    assert oracle.ts_bucket(np.array([edge - 2, edge - 1], np.int64)).tolist() == [126, 127]


def test_bucket_random_log_uniform():
    rng = np.random.default_rng(5)
    dts = np.exp(rng.uniform(0, math.log(2**40), size=400)).astype(np.int64)
    dts[::2] *= -1
    got = oracle.ts_bucket(dts)
    want = [eb.bucket_direct(int(d)) for d in dts]
    np.testing.assert_array_equal(got, want)


def test_bucket_smaller_table_clamps():
    assert oracle.ts_bucket(np.array([10**9], np.int64), num_buckets=16)[0] == 15


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------

def tiny_batch(lengths, H=2, d=4, n_max=None, cands=None, seed=0, scale=1.0):
    n_max = n_max or int(max(lengths))
    rng = np.random.default_rng(seed)
    return synth.jagged_batch(lengths, H, d, n_max, rng=rng, dtype=torch.float32,
                              num_candidates=cands, qkvu_scale=scale)


def run(b, **kw):
    return oracle.batch_attn(b, want_o=True, **kw)


# ----------------------------------------------------------------------------
# closed forms
# ----------------------------------------------------------------------------

def test_zero_scores_give_beta_times_u():
    b = tiny_batch([5, 3, 7], cands=[0, 1, 3])
    b.q.zero_()
    b.k.zero_()
    b.rab_pos[:] = 0
    b.rab_ts[:] = 0
    rng = np.random.default_rng(1)
    D = b.num_heads * b.head_dim
    b.ln_gamma = rng.normal(size=D)
    b.ln_beta = rng.normal(size=D)
    y, o = run(b)
    assert np.all(o == 0.0)
    np.testing.assert_allclose(y, b.ln_beta[None, :] * b.u.double().numpy(), rtol=0, atol=1e-15)


@pytest.mark.parametrize("cands", [None, [0, 2, 4]])
def test_constant_bias_is_masked_prefix_sum(cands):
    lengths = [6, 4, 9]
    b = tiny_batch(lengths, cands=cands, n_max=12)
    b.k.zero_()
    c_pos, c_ts = 0.7, -0.2
    b.rab_pos[:] = c_pos
    b.rab_ts[:] = c_ts
    _, o = run(b)
    w = silu(float(np.float32(c_pos)) + float(np.float32(c_ts))) / b.n_max
    v = b.v.double().numpy()
    off = b.seq_offsets
    for u in range(len(lengths)):
        n = lengths[u]
        c = 0 if cands is None else cands[u]
        h = n - c
        vs = v[off[u]:off[u + 1]]
        csum = np.cumsum(vs, axis=0)
        for i in range(n):
            if i < h:
                want = w * csum[i]
            else:
                want = w * ((csum[h - 1] if h > 0 else 0.0) + vs[i])
            np.testing.assert_allclose(o[off[u] + i], want, rtol=1e-12, atol=1e-15)


def test_single_token_user_closed_form():
    b = tiny_batch([1, 1], H=3, d=5, n_max=4, seed=3)
    _, o = run(b)
    q, k, v = (t.double().numpy() for t in (b.q, b.k, b.v))
    for r in range(2):
        for h in range(3):
            s = b.alpha * float(np.dot(q[r, h], k[r, h])) + float(b.rab_pos[b.n_max - 1]) + float(b.rab_ts[0])
            np.testing.assert_allclose(o[r, h], silu(s) / b.n_max * v[r, h], rtol=1e-13, atol=1e-16)


def test_layernorm_matches_torch():
    b = tiny_batch([7, 4], H=2, d=8, cands=[0, 2])
    rng = np.random.default_rng(2)
    D = 16
    b.ln_gamma = rng.normal(size=D)
    b.ln_beta = rng.normal(size=D)
    b.u = torch.ones_like(b.u)
    y, o = run(b)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(o.reshape(len(o), D)), (D,),
                                         torch.from_numpy(b.ln_gamma), torch.from_numpy(b.ln_beta),
                                         eps=b.ln_eps).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------
# one-hot bias probes
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("delta", [0, 1, 3, -1])
def test_one_hot_position_bias(delta):
    lengths, cands = [8, 6], [0, 3]
    b = tiny_batch(lengths, cands=cands, n_max=10)
    b.q.zero_()
    b.k.zero_()
    b.rab_ts[:] = 0
    b.rab_pos[:] = 0
    big = 3.0
    b.rab_pos[delta + b.n_max - 1] = big
    _, o = run(b)
    v = b.v.double().numpy()
    w = silu(big) / b.n_max
    for u, (n, c) in enumerate(zip(lengths, cands)):
        h = n - c
        base = b.seq_offsets[u]
        for i in range(n):
            # p(i) = min(i, h); key j contributes iff allowed and p(i) - p(j) == delta
            want = np.zeros_like(v[0])
            if i < h:
                j = i - delta
                if 0 <= j <= i:
                    want = w * v[base + j]
            else:
                if delta == 0:
                    want = w * v[base + i]                  # the candidate itself
                elif 1 <= delta <= h:
                    want = w * v[base + h - delta]          # shared history key
            np.testing.assert_allclose(o[base + i], want, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("bstar", [0, 2, 7, 9])
def test_one_hot_time_bias(bstar):
    lengths, cands = [9, 7], [0, 2]
    b = tiny_batch(lengths, cands=cands, n_max=9)
    # hand-made non-decreasing timestamps spanning several buckets
    ts = []
    for n, c in zip(lengths, cands):
        hist = [1_000_000 + int(3 ** (0.8 * j)) + j for j in range(n - c)]
        ts += hist + [hist[-1]] * c
    b.timestamps = np.array(ts, dtype=np.int64)
    b.q.zero_()
    b.k.zero_()
    b.rab_pos[:] = 0
    b.rab_ts[:] = 0
    big = 2.5
    b.rab_ts[bstar] = big
    _, o = run(b)
    v = b.v.double().numpy()
    w = silu(big) / b.n_max
    for u, (n, c) in enumerate(zip(lengths, cands)):
        h = n - c
        base = b.seq_offsets[u]
        for i in range(n):
            want = np.zeros_like(v[0])
            for j in range(n):
                ok = (j <= i) if i < h else (j < h or j == i)
                if ok and eb.bucket(ts[base + i] - ts[base + j]) == bstar:
                    want = want + w * v[base + j]
            np.testing.assert_allclose(o[base + i], want, rtol=1e-12, atol=1e-15)


# ----------------------------------------------------------------------------
# brute force over explicitly enumerated pair sets (tiny inputs)
# ----------------------------------------------------------------------------

def brute_force(b):
    q, k, v, u = (t.double().numpy() for t in (b.q, b.k, b.v, b.u))
    H, d = b.num_heads, b.head_dim
    D = H * d
    out = np.zeros((b.total_tokens, D))
    for usr in range(b.batch):
        lo, hi = int(b.seq_offsets[usr]), int(b.seq_offsets[usr + 1])
        n = hi - lo
        c = 0 if b.num_candidates is None else int(b.num_candidates[usr])
        h = n - c
        history_pairs = {(i, j) for i in range(h) for j in range(i + 1)}
        candidate_pairs = {(i, j) for i in range(h, n) for j in range(h)} | {(i, i) for i in range(h, n)}
        pairs = history_pairs | candidate_pairs
        pos = [min(i, h) for i in range(n)]
        o = np.zeros((n, H, d))
        for (i, j) in sorted(pairs):
            rel = pos[i] - pos[j]
            bias = float(b.rab_pos[rel + b.n_max - 1]) + float(b.rab_ts[eb.bucket(b.timestamps[lo + i] - b.timestamps[lo + j])])
            for hh in range(H):
                s = b.alpha * sum(q[lo + i, hh, e] * k[lo + j, hh, e] for e in range(d)) + bias
                o[i, hh] += silu(s) / b.n_max * v[lo + j, hh]
        flat = torch.from_numpy(o.reshape(n, D))
        g = None if b.ln_gamma is None else torch.from_numpy(np.asarray(b.ln_gamma, np.float64))
        bb = None if b.ln_beta is None else torch.from_numpy(np.asarray(b.ln_beta, np.float64))
        y = torch.nn.functional.layer_norm(flat, (D,), g, bb, eps=b.ln_eps).numpy() * u[lo:hi]
        out[lo:hi] = y
    return out


@pytest.mark.parametrize("lengths,cands,H,d", [
    ([1, 5, 9], None, 2, 3),
    ([4, 6], [1, 6], 1, 4),
    ([7, 2, 3], [3, 0, 1], 3, 1),
])
def test_brute_force_tiny(lengths, cands, H, d):
    b = tiny_batch(lengths, H=H, d=d, cands=cands, n_max=11, seed=sum(lengths))
    rng = np.random.default_rng(7)
    b.rab_pos = rng.normal(0, 0.5, size=2 * b.n_max - 1).astype(np.float32)
    b.rab_ts = rng.normal(0, 0.5, size=128).astype(np.float32)
    b.ln_gamma = rng.normal(size=H * d)
    b.ln_beta = rng.normal(size=H * d)
    y = oracle.batch_attn(b)
    np.testing.assert_allclose(y, brute_force(b), rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------
# invariants
# ----------------------------------------------------------------------------

def test_causality():
    b = tiny_batch([12], H=2, d=4, seed=11)
    y0 = oracle.batch_attn(b)
    i0 = 5
    for t in (b.q, b.k, b.v, b.u):
        t[i0 + 1:] = torch.randn_like(t[i0 + 1:])
    y1 = oracle.batch_attn(b)
    assert np.array_equal(y0[:i0 + 1], y1[:i0 + 1])
    assert not np.array_equal(y0[i0 + 1:], y1[i0 + 1:])


def test_jagged_batch_equals_per_user_runs():
    b = tiny_batch([6, 1, 9], H=2, d=4, cands=[2, 0, 3], seed=4)
    y = oracle.batch_attn(b)
    off = b.seq_offsets
    for usr in range(3):
        lo, hi = off[usr], off[usr + 1]
        yu = oracle.attn_jagged(b.q[lo:hi], b.k[lo:hi], b.v[lo:hi], b.u[lo:hi],
                                np.array([0, hi - lo]), b.timestamps[lo:hi], b.num_candidates[usr:usr + 1],
                                b.rab_pos, b.rab_ts, b.alpha, b.n_max)
        assert np.array_equal(y[lo:hi], yu)


def test_candidate_permutation_equivariance():
    n, c = 10, 4
    b = tiny_batch([n], H=2, d=4, cands=[c], seed=8)
    y0 = oracle.batch_attn(b)
    h = n - c
    perm = np.array(list(range(h)) + list(h + np.random.default_rng(0).permutation(c)))
    b2 = tiny_batch([n], H=2, d=4, cands=[c], seed=8)
    for name in ("q", "k", "v", "u"):
        setattr(b2, name, getattr(b, name)[perm].clone())
    b2.timestamps = b.timestamps[perm]
    y1 = oracle.batch_attn(b2)
    np.testing.assert_allclose(y1, y0[perm], rtol=1e-13, atol=1e-15)


def test_head_independence():
    b = tiny_batch([7, 5], H=3, d=4, cands=[0, 2], seed=9)
    _, o0 = run(b)
    b.q[:, 1] += 1.0
    b.k[:, 1] *= -1.0
    b.v[:, 1] += 0.5
    _, o1 = run(b)
    assert np.array_equal(o0[:, [0, 2]], o1[:, [0, 2]])
    assert not np.array_equal(o0[:, 1], o1[:, 1])


def full_recompute_inputs(pb):
    """Jagged batch holding prefix + new tokens of every user (for the paged invariant)."""
    qs, ks, vs, us, lens = [], [], [], [], []
    H, d = pb.num_heads, pb.head_dim
    for usr in range(pb.batch):
        lo, hi = pb.new_offsets[usr], pb.new_offsets[usr + 1]
        L = int(pb.cached_lens[usr])
        qs += [torch.zeros(L, H, d, dtype=pb.q.dtype), pb.q[lo:hi]]
        ks += [pb.k_prefix[usr].to(pb.k.dtype), pb.k[lo:hi]]
        vs += [pb.v_prefix[usr].to(pb.v.dtype), pb.v[lo:hi]]
        us += [torch.zeros(L, H * d, dtype=pb.u.dtype), pb.u[lo:hi]]
        lens.append(L + hi - lo)
    return (torch.cat(qs), torch.cat(ks), torch.cat(vs), torch.cat(us),
            synth.offsets_from_lengths(lens))


def test_paged_equals_full_recompute():
    rng = np.random.default_rng(12)
    pb = synth.paged_batch([37, 64, 5, 0], [3, 2, 4, 2], [2, 0, 3, 1], 2, 4, 80, rng=rng,
                           page_size=8, dtype=torch.float32)
    y_paged = oracle.batch_paged(pb)
    assert np.isfinite(y_paged).all()          # NaN-poisoned pool slots never read
    q, k, v, u, off = full_recompute_inputs(pb)
    cands = pb.num_candidates
    y_full = oracle.attn_jagged(q, k, v, u, off, pb.timestamps, cands, pb.rab_pos, pb.rab_ts,
                                pb.alpha, pb.n_max)
    rows = []
    for usr in range(pb.batch):
        L = int(pb.cached_lens[usr])
        rows += list(range(off[usr] + L, off[usr + 1]))
    assert np.array_equal(y_paged, y_full[rows])


def test_allowed_pairs_count():
    # causal user of n: n(n+1)/2 pairs; candidate block: c*h + c
    assert oracle.allowed_pairs(np.array([0, 5, 12])) == 15 + 28
    assert oracle.allowed_pairs(np.array([0, 10]), np.array([4])) == 21 + 4 * 6 + 4


# ----------------------------------------------------------------------------
# layer glue
# ----------------------------------------------------------------------------

def test_silu_special_values():
    x = np.array([0.0, 40.0, -40.0, 1.5, -1.5])
    s = olayer.silu(x)
    assert s[0] == 0.0
    assert abs(s[1] - 40.0) < 1e-12 and abs(s[2]) < 1e-15
    assert abs((s[3] - s[4]) - 1.5) < 1e-15          # silu(x) - silu(-x) = x


def test_f1_block_order():
    rng = np.random.default_rng(3)
    H, d, dm = 2, 3, 5
    x = rng.normal(size=(4, dm))
    w = synth.layer_weights(rng, dm, H, d)
    u, v, q, k = olayer.f1(x, w.w1, w.b1, H, d)
    hd = H * d
    for blk, out in enumerate([u, v.reshape(4, hd), q.reshape(4, hd), k.reshape(4, hd)]):
        w2 = w.w1.copy()
        w2[:, blk * hd:(blk + 1) * hd] += 1.0   # perturb only this block
        outs = olayer.f1(x, w2, w.b1, H, d)
        changed = [not np.array_equal(a.reshape(4, hd), b.reshape(4, hd))
                   for a, b in zip(outs, [u, v, q, k])]
        assert changed == [i == blk for i in range(4)]
    # head-major inside a block: head 1 of q is columns 2*hd + d .. 2*hd + 2d
    w3 = w.w1.copy()
    w3[:, 2 * hd + d:2 * hd + 2 * d] = 0.0
    _, _, q3, _ = olayer.f1(x, w3, w.b1, H, d)
    assert np.all(q3[:, 1] == 0.0) and np.array_equal(q3[:, 0], q[:, 0])


def test_f2_orientation_with_permutation_and_one_hot_weights():
    # f2 maps y [T, H*d] to x_next [T, d_model] as x_next[t, m] = sum_f y[t, f] W2[f, m] + b2[m].
    # A permutation W2 (W2[f, m] = 1 iff m = perm[f]) must move feature f of y to
    # output column perm[f]; the transposed matrix would apply the inverse
    # permutation instead, which differs for a permutation with no symmetry.
    rng = np.random.default_rng(11)
    T, F = 6, 8
    y = rng.normal(size=(T, F))
    perm = np.array([3, 0, 6, 1, 7, 2, 5, 4])
    assert not np.array_equal(perm, np.argsort(perm))      # not its own inverse
    w2 = np.zeros((F, F))
    w2[np.arange(F), perm] = 1.0
    b2 = np.arange(F, dtype=np.float64) * 10.0
    want = np.empty((T, F))
    for f in range(F):
        want[:, perm[f]] = y[:, f]
    want += b2
    np.testing.assert_array_equal(olayer.f2(y, w2, b2), want)
    # a one-hot weight picks one feature into one output column (d_model != H*d)
    w1hot = np.zeros((F, 3))
    w1hot[5, 2] = 2.0
    out = olayer.f2(y, w1hot, np.zeros(3))
    np.testing.assert_array_equal(out[:, 2], 2.0 * y[:, 5])
    assert np.all(out[:, :2] == 0.0)
