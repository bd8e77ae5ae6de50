"""M-FALCON scoring of candidate sets against a cached history, in
microbatches: equal to the oracle's paged attention with every new token a
candidate, independent of the microbatch size, and failures reported."""
import numpy as np
import pytest
import torch

import generative_recommender_attention_jagged_b200 as hstu
import oracle
import synth

from .gpu_helpers import BF16_TOL, F32_TOL, dev, host64, rel_err

pytestmark = pytest.mark.gpu


def candidate_batch(cached, cands, seed, dtype=torch.bfloat16, H=4, d=128, n_max=1024):
    rng = np.random.default_rng(seed)
    # no new actions: the new tokens are the candidates, which share the last history timestamp
    return synth.paged_batch(cached, 0, cands, H, d, n_max, rng=rng, dtype=dtype, spare_pages=3)


def split_timestamps(pb):
    hist, hist_off, cand = [], [0], []
    for b in range(pb.batch if hasattr(pb, "batch") else len(pb.cached_lens)):
        L = int(pb.cached_lens[b])
        t = pb.timestamps[pb.ts_offsets[b]:pb.ts_offsets[b + 1]]
        hist.append(t[:L])
        cand.append(t[L:])
        hist_off.append(hist_off[-1] + L)
    return (np.concatenate(hist).astype(np.int64), np.array(hist_off, np.int32),
            np.concatenate(cand).astype(np.int64))


def run_mfalcon(pb, microbatch, num_splits=None, force_simt=False):
    hist, hist_off, cand_ts = split_timestamps(pb)
    max_c = int(np.max(np.diff(pb.new_offsets))) if len(pb.new_offsets) > 1 else 0
    out, ws = hstu.hstu_mfalcon_fwd(
        dev(pb.q), dev(pb.k), dev(pb.v), dev(pb.u), dev(pb.new_offsets, torch.int32), dev(hist, torch.int64),
        dev(hist_off, torch.int32), dev(cand_ts, torch.int64), dev(pb.rab_pos, torch.float32),
        dev(pb.rab_ts, torch.float32), dev(pb.k_pool), dev(pb.v_pool), dev(pb.kv_page_table, torch.int32),
        dev(pb.cached_lens, torch.int32), n_max=pb.n_max, alpha=pb.alpha, microbatch=microbatch,
        max_candidates=max_c, max_cached_len=int(np.max(pb.cached_lens)), num_splits=num_splits,
        force_simt=force_simt)
    status = hstu.hstu_check_device_error(ws)
    return out, status


@pytest.mark.parametrize("microbatch", [32, 100, 128, 300])
def test_matches_oracle(microbatch):
    pb = candidate_batch([300, 129, 64, 520], [257, 0, 50, 130], seed=microbatch)
    out, status = run_mfalcon(pb, microbatch)
    assert status == 0
    want = oracle.batch_paged(pb)
    assert rel_err(host64(out), want) <= BF16_TOL


def test_microbatch_size_does_not_change_outputs():
    # each row is computed from its own q, k, v and the history only: with one
    # key split the outputs are bit-identical whatever the packing
    pb = candidate_batch([200, 333], [300, 77], seed=5)
    a, s1 = run_mfalcon(pb, 64, num_splits=1)
    b, s2 = run_mfalcon(pb, 200, num_splits=1)
    assert s1 == s2 == 0
    assert torch.equal(a, b)


def test_fp32_path_matches_oracle():
    pb = candidate_batch([40, 17], [21, 9], seed=7, dtype=torch.float32, H=2, d=32, n_max=128)
    out, status = run_mfalcon(pb, 8, force_simt=True)
    assert status == 0
    assert rel_err(host64(out), oracle.batch_paged(pb)) <= F32_TOL


def test_microbatch_over_n_max_is_reported():
    pb = candidate_batch([900], [200], seed=9, n_max=1024)
    _, status = run_mfalcon(pb, 200)             # 900 + 200 > n_max
    assert status == -4


def test_bad_candidate_offsets_are_reported():
    pb = candidate_batch([100, 50], [20, 10], seed=11)
    pb.new_offsets = np.array([0, 25, 30], np.int64)  # user 0 claims more candidates than max_candidates
    hist, hist_off, cand_ts = split_timestamps(pb)
    out, ws = hstu.hstu_mfalcon_fwd(
        dev(pb.q), dev(pb.k), dev(pb.v), dev(pb.u), dev(pb.new_offsets, torch.int32), dev(hist, torch.int64),
        dev(hist_off, torch.int32), dev(cand_ts, torch.int64), dev(pb.rab_pos, torch.float32),
        dev(pb.rab_ts, torch.float32), dev(pb.k_pool), dev(pb.v_pool), dev(pb.kv_page_table, torch.int32),
        dev(pb.cached_lens, torch.int32), n_max=pb.n_max, microbatch=16, max_candidates=20)
    assert hstu.hstu_check_device_error(ws) == -4
