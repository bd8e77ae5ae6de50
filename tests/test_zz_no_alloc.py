"""The allocation-free entry point hstu_attn_fwd_static_ws.

Some callers cannot allocate device memory where they run attention (a server
whose memory plan forbids allocation on the request path, a plug-in whose host
runtime owns the allocator).  For them the library keeps its scratch in one
16 MiB device array.  These tests call that entry point through the C ABI and
compare it with hstu_attn_fwd given a caller workspace.  Both run the same
kernels on the same work list, so the outputs must be bit-identical.  The
array keeps the previous call's contents: a larger, different problem runs
through it first, then the case under test twice, so stale work-list entries
or partial sums would show.  This file is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import generative_recommender_attention_jagged_b200 as hstu
from generative_recommender_attention_jagged_b200 import _lib
import synth
from tests.gpu_helpers import dev, run_jagged

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from generative_recommender_attention_jagged_b200 import build
    build.build()
    return _lib.load()


def call_static(lib, b, out):
    """One call through the C ABI on the current stream; returns the status."""
    T, H, d = b.q.shape
    p = hstu.attn_params(batch=b.batch, num_heads=H, head_dim=d, n_max=b.n_max, total_tokens=T,
                         max_seq_len=b.max_seq_len, dtype=b.q.dtype, alpha=b.alpha,
                         num_ts_buckets=len(b.rab_ts))
    t = {k: dev(v) for k, v in dict(q=b.q, k=b.k, v=b.v, u=b.u).items()}
    off, ts = dev(b.seq_offsets, torch.int32), dev(b.timestamps, torch.int64)
    cand = dev(b.num_candidates, torch.int32)
    rp, rt = dev(b.rab_pos, torch.float32), dev(b.rab_ts, torch.float32)
    ptr = lambda x: None if x is None else ctypes.c_void_p(x.data_ptr())
    rc = lib.hstu_attn_fwd_static_ws(ctypes.byref(p), ptr(t["q"]), ptr(t["k"]), ptr(t["v"]), ptr(t["u"]),
                                     ptr(off), ptr(ts), ptr(cand), ptr(rp), ptr(rt), None, None, ptr(out),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return rc


def static_status(lib):
    return lib.hstu_static_ws_check_device_error(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def run_static(lib, b):
    T, H, d = b.q.shape
    out = torch.full((T, H * d), float("nan"), dtype=b.q.dtype, device="cuda")
    assert call_static(lib, b, out) == 0
    assert static_status(lib) == 0
    return out.cpu()


@pytest.mark.parametrize("case", ["bf16_candidates", "fp32_tiny"])
def test_static_ws_is_bit_identical_to_workspace_entry_point(lib, case):
    # a larger, different problem first: it fills most of the 16 MiB with its
    # own work list and partial sums (about 7,200 tokens, candidates)
    big = synth.jagged_batch([3000, 2500, 1700], 4, 128, 3100, rng=np.random.default_rng(5),
                             num_candidates=[200, 0, 900])
    assert hstu.hstu_attn_workspace_size(hstu.attn_params(
        batch=3, num_heads=4, head_dim=128, n_max=3100, total_tokens=big.total_tokens, max_seq_len=3000,
        dtype=torch.bfloat16)) > 12 << 20
    assert torch.equal(run_static(lib, big), run_jagged(big).cpu())
    if case == "bf16_candidates":
        b = synth.jagged_batch([700, 130, 64, 1], 4, 128, 1024, rng=np.random.default_rng(77),
                               num_candidates=[100, 0, 64, 0])
    else:
        b = synth.workload_attention("tiny_fp32")
    want = run_jagged(b).cpu()
    for _ in range(2):
        assert torch.equal(run_static(lib, b), want)


def test_static_ws_reports_device_errors(lib):
    # unsorted timestamps: the device check fires, the status reader sees it,
    # and the next valid call starts from a cleared status word
    b = synth.jagged_batch([200, 100], 4, 128, 256, rng=np.random.default_rng(8))
    bad = synth.jagged_batch([200, 100], 4, 128, 256, rng=np.random.default_rng(8))
    bad.timestamps = bad.timestamps.copy()
    bad.timestamps[250] = bad.timestamps[249] - 5
    out = torch.empty(b.total_tokens, 512, dtype=torch.bfloat16, device="cuda")
    assert call_static(lib, bad, out) == 0          # host checks pass; the device finds the error
    assert static_status(lib) == -8                 # HSTU_ERR_UNSORTED
    assert torch.equal(run_static(lib, b), run_jagged(b).cpu())


def test_static_ws_rejects_problems_over_its_capacity(lib):
    # about 8,000 tokens at H*d = 512 fit in the 16 MiB scratch; 20,000 do not
    b = synth.jagged_batch([10000, 10000], 4, 128, 10000, rng=np.random.default_rng(3))
    out = torch.empty(b.total_tokens, 512, dtype=torch.bfloat16, device="cuda")
    assert call_static(lib, b, out) == -5  # HSTU_ERR_WORKSPACE, nothing launched
