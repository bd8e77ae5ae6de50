"""The allocation-free entry point hstu_attn_fwd_static_ws.

Some callers cannot allocate device memory where they run attention (a server
whose memory plan forbids allocation on the request path, a plug-in whose host
runtime owns the allocator).  For them the library keeps its scratch in one
16 MiB device array.  These tests call that entry point through the C ABI and
check it against hstu_attn_fwd with a caller workspace, on two calls in a row
(the array keeps the previous call's contents, so the second call shows that
whatever must start at zero is cleared).  This file is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import generative_recommender_attention_jagged_b200 as hstu
from generative_recommender_attention_jagged_b200 import _lib
import synth
from tests.gpu_helpers import BF16_TOL, F32_TOL, dev, rel_err, run_jagged

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from generative_recommender_attention_jagged_b200 import build
    build.build()
    lib = _lib.load()
    lib.hstu_attn_fwd_static_ws.argtypes = [ctypes.POINTER(_lib.AttnParams)] + [ctypes.c_void_p] * 13
    lib.hstu_attn_fwd_static_ws.restype = ctypes.c_int
    return lib


def call_static(lib, b, out):
    """One call through the C ABI; returns the status."""
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


@pytest.mark.parametrize("case", ["bf16_candidates", "fp32_tiny"])
def test_static_ws_matches_workspace_entry_point_twice(lib, case):
    if case == "bf16_candidates":
        b = synth.jagged_batch([700, 130, 64, 1], 4, 128, 1024, rng=np.random.default_rng(77),
                               num_candidates=[100, 0, 64, 0])
        tol = BF16_TOL
    else:
        b = synth.workload_attention("tiny_fp32")
        tol = F32_TOL
    want = run_jagged(b).float().cpu().numpy()
    T, H, d = b.q.shape
    for _ in range(2):
        out = torch.full((T, H * d), float("nan"), dtype=b.q.dtype, device="cuda")
        assert call_static(lib, b, out) == 0
        got = out.float().cpu().numpy()
        assert np.isfinite(got).all()
        assert rel_err(got, want) <= tol


def test_static_ws_rejects_problems_over_its_capacity(lib):
    # about 8,000 tokens at H*d = 512 fit in the 16 MiB scratch; 20,000 do not
    b = synth.jagged_batch([10000, 10000], 4, 128, 10000, rng=np.random.default_rng(3))
    out = torch.empty(b.total_tokens, 512, dtype=torch.bfloat16, device="cuda")
    assert call_static(lib, b, out) == -5  # HSTU_ERR_WORKSPACE, nothing launched
