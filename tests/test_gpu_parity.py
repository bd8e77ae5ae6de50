"""GPU parity: the CUDA library through its C ABI against the fp64 oracle.

Bar: bucket indices bit-exact; max-abs-err / max|Y| <= 1e-5 for fp32 inputs
and <= 2e-2 for bf16 inputs.  Small cases compare every element; the full
workload sizes compare sampled rows the oracle evaluates one by one, in the
same launch configuration the bench times.
"""
import math

import numpy as np
import pytest
import torch

import generative_recommender_attention_jagged_b200 as hstu
import oracle
import synth
from tests import exact_bucket as eb
from tests.gpu_helpers import (BF16_TOL, F32_TOL, dev, host64, rel_err, run_jagged, run_paged,
                               sample_rows)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from generative_recommender_attention_jagged_b200 import build
    build.build()


def small_batch(lengths, *, cands=None, H=4, d=128, n_max=None, seed=0, dtype=torch.bfloat16, scale=1.0):
    rng = np.random.default_rng(seed)
    n_max = n_max or max(8, int(max(lengths)))
    return synth.jagged_batch(lengths, H, d, n_max, rng=rng, dtype=dtype, num_candidates=cands,
                              qkvu_scale=scale)


# ----------------------------------------------------------------------------
# time buckets
# ----------------------------------------------------------------------------

def test_bucket_kernel_bit_exact_at_thresholds():
    thr = eb.integer_thresholds()
    xs = sorted({max(1, t + dl) for t in thr for dl in range(-2, 3) if t + dl - 1 < 2**63})
    dts = np.array([x - 1 for x in xs] + [-(x - 1) for x in xs] + [2**63 - 1, -(2**63)], dtype=np.int64)
    got = hstu.hstu_ts_bucket(dev(dts)).cpu().numpy()
    want = np.array([eb.bucket(int(x)) for x in dts])
    np.testing.assert_array_equal(got, want)


def test_bucket_kernel_matches_oracle_random():
    rng = np.random.default_rng(3)
    n = (1 << 20) + 17  # ragged tail
    dts = np.exp(rng.uniform(0, math.log(2.0**62), size=n)).astype(np.int64)
    dts[::3] *= -1
    got = hstu.hstu_ts_bucket(dev(dts)).cpu().numpy()
    np.testing.assert_array_equal(got, oracle.ts_bucket(dts))


@pytest.mark.parametrize("nb", [1, 16, 128])
def test_bucket_kernel_clamps_to_table(nb):
    dts = np.array([0, 5, 10**6, 10**15], dtype=np.int64)
    got = hstu.hstu_ts_bucket(dev(dts), num_buckets=nb).cpu().numpy()
    np.testing.assert_array_equal(got, oracle.ts_bucket(dts, nb))


def test_bucket_kernel_empty():
    out = hstu.hstu_ts_bucket(torch.zeros(0, dtype=torch.int64, device="cuda"))
    assert out.numel() == 0


# ----------------------------------------------------------------------------
# fp32 (CUDA-core kernel)
# ----------------------------------------------------------------------------

def test_tiny_fp32_workload_full():
    b = synth.workload_attention("tiny_fp32")
    y = host64(run_jagged(b))
    assert rel_err(y, oracle.batch_attn(b)) <= F32_TOL


def test_tiny_fp32_raw_av_and_candidates():
    b = small_batch([37, 64, 1, 20], cands=[5, 0, 1, 20], H=2, d=32, n_max=64, dtype=torch.float32,
                    scale=1 / math.sqrt(32))
    rng = np.random.default_rng(9)
    b.ln_gamma = rng.normal(size=64).astype(np.float32)
    b.ln_beta = rng.normal(size=64).astype(np.float32)
    y = host64(run_jagged(b))
    want_y, want_o = oracle.batch_attn(b, want_o=True)
    assert rel_err(y, want_y) <= F32_TOL
    o = host64(run_jagged(b, raw_av=True))
    assert rel_err(o, want_o) <= F32_TOL


@pytest.mark.parametrize("d", [1, 8, 33, 64, 200])
def test_fp32_odd_head_dims(d):
    # H = 4 keeps the fp32 row stride H*d a multiple of 4 elements for every d
    b = small_batch([9, 17, 3], cands=[0, 4, 0], H=4, d=d, n_max=20, dtype=torch.float32, seed=d)
    assert rel_err(host64(run_jagged(b)), oracle.batch_attn(b)) <= F32_TOL


# ----------------------------------------------------------------------------
# bf16 tensor-core kernel, small shapes: every element
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("lengths,cands", [
    ([128], None),                         # one exact tile
    ([1, 2, 127, 129, 300], None),         # ragged tails, tiny users
    ([513, 200, 64], [0, 0, 0]),           # several tiles, candidates given but zero
    ([700, 300], [100, 300]),              # candidates; a user made only of candidates
    ([260, 140, 257], [130, 7, 129]),      # candidate block across tile edges
])
def test_bf16_tensor_core_small(lengths, cands):
    b = small_batch(lengths, cands=cands, n_max=max(lengths) + 64, seed=len(lengths))
    want_y, want_o = oracle.batch_attn(b, want_o=True)
    o = host64(run_jagged(b, raw_av=True))
    assert rel_err(o, want_o) <= BF16_TOL
    y = host64(run_jagged(b))
    assert rel_err(y, want_y) <= BF16_TOL


@pytest.mark.parametrize("num_users", [3, 300])
def test_work_list_for_few_and_many_users(num_users):
    """The planner's last block builds the work list with its 256 threads in
    min(B, 256) groups: 3 users leave threads idle (256 = 3 x 85 + 1), 300
    users give one thread per group and several users per thread.  Every
    row must come out, with the lengths spanning one to several query blocks."""
    rng = np.random.default_rng(num_users)
    if num_users == 3:
        lengths, cands = [600, 1, 257], [0, 0, 57]
    else:
        lengths = rng.integers(1, 300, size=num_users)
        lengths[::37] = 520                    # a few users with two query blocks
        cands = np.where(np.arange(num_users) % 5 == 0, np.minimum(lengths, 9), 0)
    b = small_batch(list(lengths), cands=list(cands), n_max=640, seed=num_users)
    want_y, want_o = oracle.batch_attn(b, want_o=True)
    o = host64(run_jagged(b, raw_av=True))
    assert rel_err(o, want_o) <= BF16_TOL
    assert np.abs(o.reshape(o.shape[0], -1)).sum(axis=1).min() > 0   # no row left out of the work list


@pytest.mark.parametrize("lengths,cands", [
    ([0, 300, 0, 129, 0], [0, 40, 0, 0, 0]),   # empty users first, between and last
    ([0, 0], None),                            # an empty batch (T = 0)
])
def test_zero_length_users(lengths, cands):
    b = small_batch(lengths, cands=cands, n_max=320, seed=3)
    T = int(sum(lengths))
    y = run_jagged(b)
    assert tuple(y.shape) == (T, 4 * 128)
    if T:
        assert rel_err(host64(y), oracle.batch_attn(b)) <= BF16_TOL


def test_bf16_tensor_core_matches_cuda_core_kernel():
    b = small_batch([400, 131, 77], cands=[50, 0, 3], n_max=512, seed=5)
    o_tc = host64(run_jagged(b, raw_av=True))
    o_simt = host64(run_jagged(b, raw_av=True, force_simt=True))
    assert rel_err(o_tc, o_simt) <= BF16_TOL
    _, want_o = oracle.batch_attn(b, want_o=True)
    assert rel_err(o_simt, want_o) <= 1e-4  # fp32 math on bf16 inputs


def test_bf16_gamma_beta_and_strided_views():
    # q/k/v/u as column blocks of one [T, 4*H*d] buffer, as the layer's f1 output is laid out
    b = small_batch([300, 45], cands=[20, 0], n_max=400, seed=11)
    rng = np.random.default_rng(1)
    b.ln_gamma = rng.normal(size=512).astype(np.float32)
    b.ln_beta = rng.normal(size=512).astype(np.float32)
    T = b.total_tokens
    big = torch.cat([b.u.view(T, 512), b.v.view(T, 512), b.q.view(T, 512), b.k.view(T, 512)], 1).cuda()
    u, v, q, k = (big[:, i * 512:(i + 1) * 512] for i in range(4))
    out = hstu.hstu_attn_fwd(q.view(T, 4, 128), k.view(T, 4, 128), v.view(T, 4, 128), u,
                             dev(b.seq_offsets, torch.int32), dev(b.timestamps, torch.int64),
                             dev(b.rab_pos, torch.float32), dev(b.rab_ts, torch.float32), n_max=b.n_max,
                             num_candidates=dev(b.num_candidates, torch.int32),
                             ln_gamma=dev(b.ln_gamma), ln_beta=dev(b.ln_beta))
    torch.cuda.synchronize()
    assert rel_err(host64(out), oracle.batch_attn(b)) <= BF16_TOL


def test_bf16_larger_bias_magnitudes():
    # biases of order 1 exercise the bucket walk and position window far from zero
    b = small_batch([1000, 333], cands=[0, 33], n_max=1400, seed=21)
    rng = np.random.default_rng(2)
    b.rab_pos = rng.normal(0, 1.0, size=2 * b.n_max - 1).astype(np.float32)
    b.rab_ts = rng.normal(0, 1.0, size=128).astype(np.float32)
    _, want_o = oracle.batch_attn(b, want_o=True)
    assert rel_err(host64(run_jagged(b, raw_av=True)), want_o) <= BF16_TOL


def test_one_hot_time_bias_selects_exact_buckets():
    # with q = k = 0 and rab_pos = 0, only keys in the one-hot bucket contribute:
    # any bucket error on the GPU shows up as a whole missing/extra v row
    b = small_batch([600, 250], n_max=700, seed=4)
    b.q.zero_()
    b.k.zero_()
    b.rab_pos[:] = 0
    for bstar in (19, 23, 30):
        b.rab_ts[:] = 0
        b.rab_ts[bstar] = 4.0
        _, want_o = oracle.batch_attn(b, want_o=True)
        got = host64(run_jagged(b, raw_av=True))
        assert rel_err(got, want_o) <= 1e-2, bstar


# ----------------------------------------------------------------------------
# time buckets inside the attention kernels: wide gaps, the clamp, small tables
# ----------------------------------------------------------------------------

def wide_gap_timestamps(rng, lengths, cands=None):
    """Non-decreasing timestamps whose gaps mix 1-4 s steps, ~600 s steps and
    jumps of 2^10 .. 2^32 and 2^32 .. 2^52 s, so that every bucket range
    occurs.  One 32-key chunk then crosses several bucket edges while
    |dt| + 1 >= 2^32 (the kernels' per-column walk), and pairs far apart reach
    |dt| + 1 >= e^(0.301*127) ~ 2^55.1, the last bucket (the clamp)."""
    out = []
    for i, n in enumerate(lengths):
        c = 0 if cands is None else int(cands[i])
        h = int(n) - c
        m = max(h - 1, 0)
        kind = rng.choice(4, size=m, p=[0.2, 0.3, 0.2, 0.3])
        tiny = rng.integers(1, 5, size=m)
        small = np.maximum(1, np.rint(rng.exponential(600.0, size=m)))
        medium = np.rint(np.exp2(rng.uniform(10, 32, size=m)))
        big = np.rint(np.exp2(rng.uniform(32, 52, size=m)))
        gaps = np.choose(kind, [tiny, small, medium, big]).astype(np.int64)
        t0 = -(1 << 60) + int(rng.integers(0, 1 << 40))
        hist = t0 + np.concatenate([np.zeros(1 if h > 0 else 0, np.int64), np.cumsum(gaps)])
        last = hist[-1] if h > 0 else t0
        out.append(np.concatenate([hist, np.full(c, last, dtype=np.int64)]))
    ts = np.concatenate(out)
    assert np.abs(ts).max() < (1 << 61)  # the library's timestamp range
    return ts


def wide_gap_batch(nb, *, seed, dtype=torch.bfloat16, d=128, H=4):
    lengths, cands = [1100, 300, 77, 260], [0, 40, 0, 130]
    b = small_batch(lengths, cands=cands, H=H, d=d, n_max=1200, seed=seed, dtype=dtype,
                    scale=1.0 if dtype == torch.bfloat16 else 1 / math.sqrt(d))
    b.timestamps = wide_gap_timestamps(np.random.default_rng(seed + 100), lengths, cands)
    rng = np.random.default_rng(seed + 200)
    b.rab_ts = rng.normal(0, 0.5, size=nb).astype(np.float32)   # order-1 entries: a wrong bucket shows
    return b


def test_wide_gap_timestamps_reach_walk_mode_and_clamp():
    # the inputs below really exercise what they claim (checked on the host
    # with the oracle's bucket rule)
    b = wide_gap_batch(128, seed=1)
    ts, off = b.timestamps, b.seq_offsets
    lo, hi = int(off[0]), int(off[1])
    t = ts[lo:hi]
    dt = t[-1] - t[:64]
    assert (oracle.ts_bucket(dt) == 127).all()                   # far pairs clamp
    multi_edge_wide = 0
    for i in range(200, hi - lo, 37):
        for c0 in range(0, i - 32, 32):
            d = t[i] - t[c0:c0 + 32]
            bk = oracle.ts_bucket(d)
            if len(set(bk.tolist())) > 2 and (d.min() + 1) >= 2 ** 32:
                multi_edge_wide += 1
    assert multi_edge_wide > 20


@pytest.mark.parametrize("nb", [1, 16, 100, 128])
def test_wide_gaps_and_bucket_tables_tensor_core(nb):
    b = wide_gap_batch(nb, seed=nb)
    want_y, want_o = oracle.batch_attn(b, want_o=True)
    o = host64(run_jagged(b, raw_av=True))
    assert rel_err(o, want_o) <= BF16_TOL
    y = host64(run_jagged(b))
    assert rel_err(y, want_y) <= BF16_TOL


@pytest.mark.parametrize("nb", [1, 16, 100, 128])
def test_wide_gaps_and_bucket_tables_cuda_core(nb):
    b = wide_gap_batch(nb, seed=nb + 7, dtype=torch.float32, d=32, H=2)
    assert rel_err(host64(run_jagged(b)), oracle.batch_attn(b)) <= F32_TOL
    b16 = wide_gap_batch(nb, seed=nb + 9)
    _, want_o = oracle.batch_attn(b16, want_o=True)
    assert rel_err(host64(run_jagged(b16, raw_av=True, force_simt=True)), want_o) <= 1e-4


@pytest.mark.parametrize("nb,bstar", [(128, 127), (128, 100), (128, 70), (128, 44), (100, 99), (16, 15),
                                      (16, 5), (1, 0)])
@pytest.mark.parametrize("force_simt", [False, True])
def test_one_hot_time_bias_wide_gaps(nb, bstar, force_simt):
    # q = k = 0 and rab_pos = 0: only keys whose (clamped) bucket is bstar
    # contribute, so one wrong bucket anywhere is a whole v row missing or extra
    b = wide_gap_batch(nb, seed=3 * bstar + nb)
    b.q.zero_()
    b.k.zero_()
    b.rab_pos[:] = 0
    b.rab_ts[:] = 0
    b.rab_ts[bstar] = 4.0
    _, want_o = oracle.batch_attn(b, want_o=True)
    assert np.abs(want_o).max() > 0
    got = host64(run_jagged(b, raw_av=True, force_simt=force_simt))
    assert rel_err(got, want_o) <= 1e-2


def test_paged_wide_gap_timestamps():
    rng = np.random.default_rng(41)
    cached, acts, cands = [900, 300], [64, 10], [64, 5]
    pb = synth.paged_batch(cached, acts, cands, 4, 128, 1100, rng=rng)
    lengths = [c + a + k for c, a, k in zip(cached, acts, cands)]
    pb.timestamps = wide_gap_timestamps(np.random.default_rng(42), lengths, cands)
    pb.rab_ts = np.random.default_rng(43).normal(0, 0.5, size=128).astype(np.float32)
    want_y, want_o = oracle.batch_paged(pb, want_o=True)
    assert rel_err(host64(run_paged(pb, raw_av=True, num_splits=2)), want_o) <= BF16_TOL
    assert rel_err(host64(run_paged(pb, num_splits=2)), want_y) <= BF16_TOL


# ----------------------------------------------------------------------------
# invariants on the GPU
# ----------------------------------------------------------------------------

def test_gpu_causality_bitwise():
    b = small_batch([520], n_max=600, seed=7)
    y0 = run_jagged(b).cpu()
    i0 = 300
    for t in (b.q, b.k, b.v, b.u):
        t[i0 + 1:] = torch.randn_like(t[i0 + 1:].float()).to(t.dtype)
    y1 = run_jagged(b).cpu()
    assert torch.equal(y0[:i0 + 1], y1[:i0 + 1])
    assert not torch.equal(y0[i0 + 1:], y1[i0 + 1:])


def test_gpu_jagged_batch_equals_per_user_runs():
    b = small_batch([300, 129, 1, 450], cands=[0, 9, 0, 60], n_max=500, seed=8)
    y = run_jagged(b).cpu()
    off = b.seq_offsets
    for u in range(b.batch):
        lo, hi = int(off[u]), int(off[u + 1])
        bu = synth.JaggedBatch(q=b.q[lo:hi], k=b.k[lo:hi], v=b.v[lo:hi], u=b.u[lo:hi],
                               seq_offsets=np.array([0, hi - lo], np.int32), timestamps=b.timestamps[lo:hi],
                               num_candidates=b.num_candidates[u:u + 1], rab_pos=b.rab_pos, rab_ts=b.rab_ts,
                               alpha=b.alpha, n_max=b.n_max, num_heads=b.num_heads, head_dim=b.head_dim)
        assert torch.equal(run_jagged(bu).cpu(), y[lo:hi]), u


def test_gpu_candidate_permutation_equivariance():
    n, c = 400, 150
    b = small_batch([n], cands=[c], n_max=512, seed=10)
    y0 = host64(run_jagged(b))
    h = n - c
    perm = np.array(list(range(h)) + list(h + np.random.default_rng(0).permutation(c)))
    for name in ("q", "k", "v", "u"):
        setattr(b, name, getattr(b, name)[perm].clone())
    b.timestamps = b.timestamps[perm]
    y1 = host64(run_jagged(b))
    assert rel_err(y1, y0[perm]) <= 1e-6


# ----------------------------------------------------------------------------
# device-detected errors (the kernels' own checks; nothing out of bounds is read)
# ----------------------------------------------------------------------------

def _status(b, **kw):
    ws = torch.empty(hstu.hstu_attn_workspace_size(hstu.attn_params(
        batch=b.batch, num_heads=b.num_heads, head_dim=b.head_dim, n_max=b.n_max, total_tokens=b.total_tokens,
        max_seq_len=b.n_max, dtype=b.q.dtype)), dtype=torch.uint8, device="cuda")
    run_jagged(b, workspace=ws, **kw)
    return hstu.hstu_check_device_error(ws)


def test_device_reports_unsorted_timestamps():
    b = small_batch([200, 100], n_max=256)
    assert _status(b) == 0
    b.timestamps = b.timestamps.copy()
    b.timestamps[250] = b.timestamps[249] - 5
    assert _status(b) == -8


def test_device_reports_length_above_n_max():
    b = small_batch([200, 100], n_max=256)
    b.n_max = 150
    b.rab_pos = b.rab_pos[:2 * 150 - 1]
    assert _status(b) == -4


def test_device_reports_too_many_candidates():
    b = small_batch([200, 100], cands=[0, 5], n_max=256)
    b.num_candidates = np.array([0, 101], np.int32)
    assert _status(b) == -4


# ----------------------------------------------------------------------------
# paged incremental mode
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("cached,acts,cands,page,splits", [
    ([300, 128, 0, 77], [5, 64, 3, 1], [2, 64, 0, 1], 32, 1),
    ([1000, 520], [64, 1], [64, 0], 32, 3),
    ([256, 130], [10, 20], [4, 0], 64, 2),
    ([511, 129], [100, 140], [28, 0], 128, 4),
])
def test_paged_small_matches_oracle(cached, acts, cands, page, splits):
    rng = np.random.default_rng(sum(cached))
    n_max = max(c + a + k for c, a, k in zip(cached, acts, cands)) + 16
    pb = synth.paged_batch(cached, acts, cands, 4, 128, n_max, rng=rng, page_size=page)
    want_y, want_o = oracle.batch_paged(pb, want_o=True)
    o = host64(run_paged(pb, raw_av=True, num_splits=splits))
    assert np.isfinite(o).all()  # the NaN-poisoned pool slots are never read into the result
    assert rel_err(o, want_o) <= BF16_TOL
    y = host64(run_paged(pb, num_splits=splits))
    assert rel_err(y, want_y) <= BF16_TOL


def test_paged_cuda_core_kernel_matches_oracle():
    rng = np.random.default_rng(5)
    pb = synth.paged_batch([100, 37], [6, 3], [2, 1], 2, 64, 160, rng=rng, page_size=16, dtype=torch.float32)
    assert rel_err(host64(run_paged(pb, force_simt=True)), oracle.batch_paged(pb)) <= F32_TOL


def test_paged_equals_full_recompute_on_gpu():
    rng = np.random.default_rng(6)
    pb = synth.paged_batch([700, 333], [64, 10], [64, 5], 4, 128, 900, rng=rng)
    y_paged = host64(run_paged(pb, num_splits=2))
    qs, ks, vs, us, lens = [], [], [], [], []
    for u in range(pb.batch):
        lo, hi = pb.new_offsets[u], pb.new_offsets[u + 1]
        L = int(pb.cached_lens[u])
        qs += [torch.zeros(L, 4, 128, dtype=torch.bfloat16), pb.q[lo:hi]]
        ks += [pb.k_prefix[u], pb.k[lo:hi]]
        vs += [pb.v_prefix[u], pb.v[lo:hi]]
        us += [torch.zeros(L, 512, dtype=torch.bfloat16), pb.u[lo:hi]]
        lens.append(L + hi - lo)
    full = synth.JaggedBatch(q=torch.cat(qs), k=torch.cat(ks), v=torch.cat(vs), u=torch.cat(us),
                             seq_offsets=synth.offsets_from_lengths(lens), timestamps=pb.timestamps,
                             num_candidates=pb.num_candidates, rab_pos=pb.rab_pos, rab_ts=pb.rab_ts,
                             alpha=pb.alpha, n_max=pb.n_max, num_heads=4, head_dim=128)
    y_full = host64(run_jagged(full))
    rows = np.concatenate([np.arange(full.seq_offsets[u] + pb.cached_lens[u], full.seq_offsets[u + 1])
                           for u in range(pb.batch)])
    assert rel_err(y_paged, y_full[rows]) <= BF16_TOL


def test_device_reports_bad_page_id():
    rng = np.random.default_rng(7)
    pb = synth.paged_batch([100, 64], [4, 4], [1, 1], 4, 128, 200, rng=rng)
    pb.kv_page_table = pb.kv_page_table.copy()
    pb.kv_page_table[1, 0] = pb.k_pool.shape[0] + 3
    params = hstu.attn_params(batch=2, num_heads=4, head_dim=128, n_max=200, total_tokens=int(pb.new_offsets[-1]),
                              max_seq_len=200, dtype=torch.bfloat16)
    ws = torch.empty(hstu.hstu_attn_paged_workspace_size(params, 2), dtype=torch.uint8, device="cuda")
    run_paged(pb, num_splits=2, workspace=ws)
    assert hstu.hstu_check_device_error(ws) == -9


# ----------------------------------------------------------------------------
# full workload sizes: sampled rows, the bench's launch configuration
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["layer_bf16", "stack8_bf16", "mfalcon_bf16"])
def test_workload_sampled_rows(name):
    b = synth.workload_attention(name, layer=0)
    y = host64(run_jagged(b))
    assert np.isfinite(y).all()
    rows = sample_rows(b.seq_offsets, b.num_candidates, per_user=4)
    want = oracle.batch_attn(b, rows=rows)
    assert rel_err(y[rows], want) <= BF16_TOL


def test_paged_workload_sampled_rows():
    pb = synth.workload_paged(layer=0)
    y = host64(run_paged(pb))
    assert np.isfinite(y).all()
    rows = sample_rows(pb.new_offsets, pb.num_candidates, per_user=6)
    want = oracle.batch_paged(pb, rows=rows)
    assert rel_err(y[rows], want) <= BF16_TOL


def test_tensor_core_path_is_the_one_that_runs():
    # the two kernels round differently (bf16 P and tanh.approx vs fp32 expf), so
    # bitwise-different outputs show the bf16 d=128 call did not take the CUDA-core kernel
    b = small_batch([300], n_max=320, seed=12)
    o_tc = run_jagged(b, raw_av=True).cpu()
    o_simt = run_jagged(b, raw_av=True, force_simt=True).cpu()
    assert not torch.equal(o_tc, o_simt)
    assert rel_err(host64(o_tc), host64(o_simt)) <= BF16_TOL


@pytest.mark.parametrize("precise", [False, True])
def test_silu_paths_both_within_tolerance(precise):
    # default: packed bf16x2 tanh/FMA; precise: fp32 tanh per score
    b = small_batch([900, 400, 129], cands=[0, 100, 0], n_max=1024, seed=31)
    rng = np.random.default_rng(4)
    b.rab_pos = rng.normal(0, 0.5, size=2 * b.n_max - 1).astype(np.float32)
    b.rab_ts = rng.normal(0, 0.5, size=128).astype(np.float32)
    want_y, want_o = oracle.batch_attn(b, want_o=True)
    o = host64(run_jagged(b, raw_av=True, precise_silu=precise))
    y = host64(run_jagged(b, precise_silu=precise))
    assert rel_err(o, want_o) <= BF16_TOL
    assert rel_err(y, want_y) <= BF16_TOL
