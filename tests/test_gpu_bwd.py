"""GPU backward of the attention core against the fp64 backward oracle
(itself pinned by finite differences of the forward oracle)."""
import numpy as np
import pytest
import torch

import generative_recommender_attention_jagged_b200 as hstu
import synth
from oracle import backward as obwd

from .gpu_helpers import dev, rel_err

pytestmark = pytest.mark.gpu

# The CUDA-core backward runs in fp32 on the same rounded inputs the oracle
# upcasts; a gradient entry sums up to N_max terms, so fp32 rounding stays well
# below 1e-4 of the largest entry.
BWD_TOL = 1e-4
# The tensor-core backward (bf16 inputs, d = 128) feeds its GEMMs bf16
# operands: d_o, the weights a and the score gradients ds are each rounded to
# bf16 (relative 2^-9) before fp32 accumulation, and the sigmoid comes from
# tanh.approx; the bf16 tolerance of the forward applies.
BWD_TOL_TC = 2e-2


def run(b, seed, force_simt=False):
    rng = np.random.default_rng(seed)
    g = rng.standard_normal(tuple(b.q.shape)).astype(np.float32)
    dq, dk, dv, drp, drt, ws = hstu.hstu_attn_bwd(
        dev(b.q), dev(b.k), dev(b.v), dev(b.seq_offsets, torch.int32), dev(b.timestamps, torch.int64),
        dev(b.rab_pos, torch.float32), dev(b.rab_ts, torch.float32), dev(g), n_max=b.n_max, alpha=b.alpha,
        num_candidates=dev(b.num_candidates, torch.int32), max_seq_len=b.max_seq_len, force_simt=force_simt)
    status = hstu.hstu_check_device_error(ws)
    want = obwd.attn_jagged_bwd(b.q, b.k, b.v, b.seq_offsets, b.timestamps, b.num_candidates, b.rab_pos,
                                b.rab_ts, b.alpha, b.n_max, g)
    got = [t.cpu().double().numpy() for t in (dq, dk, dv, drp, drt)]
    return status, got, want


@pytest.mark.parametrize("lengths,cands,H,d,dtype", [
    ([37, 64], None, 2, 32, torch.float32),
    ([50, 1, 77], [10, 0, 77], 2, 32, torch.float32),
    ([300, 129], [40, 0], 4, 128, torch.bfloat16),
    ([200, 65, 128], [70, 0, 1], 2, 64, torch.float32),
    ([64, 130], [64, 3], 1, 128, torch.float32),
    ([40, 9], [5, 0], 1, 48, torch.float32),       # head dim outside the tiled kernel's set
    ([0, 40, 0, 33, 0], [0, 5, 0, 0, 0], 2, 128, torch.bfloat16),   # empty users
])
def test_gradients_match_oracle(lengths, cands, H, d, dtype):
    """Default path: bf16 with d = 128 on the tensor cores, everything else on
    the fp32 CUDA-core kernels."""
    rng = np.random.default_rng(sum(lengths))
    b = synth.jagged_batch(lengths, H, d, 512, rng=rng, dtype=dtype, num_candidates=cands,
                           qkvu_scale=1.0 / np.sqrt(d) if dtype == torch.float32 else 1.0)
    status, got, want = run(b, seed=7)
    assert status == 0
    tol = BWD_TOL_TC if (dtype == torch.bfloat16 and d == 128) else BWD_TOL
    for name, gv, wv in zip(("d_q", "d_k", "d_v", "d_rab_pos", "d_rab_ts"), got, want):
        assert rel_err(gv, wv) <= tol, name


@pytest.mark.parametrize("lengths,cands,H", [
    ([300, 129], [40, 0], 4),
    ([0, 40, 0, 33, 0], [0, 5, 0, 0, 0], 2),
    ([700, 1, 257, 128], [100, 1, 0, 128], 2),     # several key and query blocks, candidates across blocks
    ([1000], [0], 1),                              # eight query blocks for key block 0
])
def test_tensor_core_gradients_match_oracle_and_fp32_path(lengths, cands, H):
    """bf16, d = 128: the tensor-core backward within the bf16 tolerance of the
    oracle, the fp32 CUDA-core kernel (force_simt) within the fp32 one."""
    rng = np.random.default_rng(sum(lengths) + 5)
    b = synth.jagged_batch(lengths, H, 128, 1024, rng=rng, dtype=torch.bfloat16, num_candidates=cands)
    status, got, want = run(b, seed=11)
    assert status == 0
    for name, gv, wv in zip(("d_q", "d_k", "d_v", "d_rab_pos", "d_rab_ts"), got, want):
        assert np.isfinite(gv).all(), name
        assert rel_err(gv, wv) <= BWD_TOL_TC, name
    status, got, _ = run(b, seed=11, force_simt=True)
    assert status == 0
    for name, gv, wv in zip(("d_q", "d_k", "d_v", "d_rab_pos", "d_rab_ts"), got, want):
        assert rel_err(gv, wv) <= BWD_TOL, name


def test_unsorted_timestamps_are_reported():
    rng = np.random.default_rng(3)
    b = synth.jagged_batch([20], 2, 32, 64, rng=rng, dtype=torch.float32)
    b.timestamps = b.timestamps.copy()
    b.timestamps[5] = b.timestamps[4] - 10
    rng2 = np.random.default_rng(0)
    g = rng2.standard_normal(tuple(b.q.shape)).astype(np.float32)
    *_, ws = hstu.hstu_attn_bwd(dev(b.q), dev(b.k), dev(b.v), dev(b.seq_offsets, torch.int32),
                                dev(b.timestamps, torch.int64), dev(b.rab_pos, torch.float32),
                                dev(b.rab_ts, torch.float32), dev(g), n_max=b.n_max, alpha=b.alpha)
    assert hstu.hstu_check_device_error(ws) == -8


def test_empty_batch():
    rng = np.random.default_rng(4)
    b = synth.jagged_batch([0, 0], 2, 64, 64, rng=rng, dtype=torch.float32)
    status, got, want = run(b, seed=1)
    assert status == 0
    for gv, wv in zip(got, want):
        assert gv.shape == wv.shape
        assert not np.any(gv)                   # no pairs: every gradient is zero
