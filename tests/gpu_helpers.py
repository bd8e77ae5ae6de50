"""Helpers for the GPU parity tests: move synth batches to the device, run
the library, compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import generative_recommender_attention_jagged_b200 as hstu

BF16_TOL = 2e-2   # max-abs-err / max|Y| for bf16 inputs
F32_TOL = 1e-5    # max-abs-err / max|Y| for fp32 inputs


def dev(x, dtype=None):
    if x is None:
        return None
    if isinstance(x, np.ndarray):
        x = torch.from_numpy(np.ascontiguousarray(x))
    if dtype is not None:
        x = x.to(dtype)
    return x.cuda()


def run_jagged(b, *, raw_av=False, force_simt=False, workspace=None, check_status=True, **kw):
    out = hstu.hstu_attn_fwd(dev(b.q), dev(b.k), dev(b.v), dev(b.u), dev(b.seq_offsets, torch.int32),
                             dev(b.timestamps, torch.int64), dev(b.rab_pos, torch.float32),
                             dev(b.rab_ts, torch.float32), n_max=b.n_max, alpha=b.alpha,
                             num_candidates=dev(b.num_candidates, torch.int32),
                             ln_gamma=dev(b.ln_gamma, torch.float32), ln_beta=dev(b.ln_beta, torch.float32),
                             ln_eps=b.ln_eps, max_seq_len=b.max_seq_len, raw_av=raw_av, force_simt=force_simt,
                             workspace=workspace, **kw)
    torch.cuda.synchronize()
    return out


def run_paged(pb, *, raw_av=False, force_simt=False, num_splits=None, workspace=None):
    out = hstu.hstu_attn_fwd_paged(
        dev(pb.q), dev(pb.k), dev(pb.v), dev(pb.u), dev(pb.new_offsets, torch.int32),
        dev(pb.timestamps, torch.int64), dev(pb.ts_offsets, torch.int32), dev(pb.rab_pos, torch.float32),
        dev(pb.rab_ts, torch.float32), dev(pb.k_pool), dev(pb.v_pool), dev(pb.kv_page_table, torch.int32),
        dev(pb.cached_lens, torch.int32), n_max=pb.n_max, alpha=pb.alpha,
        num_candidates=dev(pb.num_candidates, torch.int32), ln_gamma=dev(pb.ln_gamma, torch.float32),
        ln_beta=dev(pb.ln_beta, torch.float32), ln_eps=pb.ln_eps, num_splits=num_splits,
        max_cached_len=int(pb.cached_lens.max()) if len(pb.cached_lens) else 0, raw_av=raw_av,
        force_simt=force_simt, workspace=workspace)
    torch.cuda.synchronize()
    return out


def host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def rel_err(got: np.ndarray, want: np.ndarray) -> float:
    got = np.asarray(got, np.float64).reshape(want.shape)
    scale = float(np.max(np.abs(want)))
    if scale == 0.0:
        return float(np.max(np.abs(got)))
    return float(np.max(np.abs(got - want))) / scale


def sample_rows(seq_offsets, num_candidates=None, per_user: int = 6, seed: int = 0):
    """A few rows per user: first, last, tile edges, candidates, random ones."""
    rng = np.random.default_rng(seed)
    rows = []
    off = np.asarray(seq_offsets)
    for u in range(len(off) - 1):
        lo, hi = int(off[u]), int(off[u + 1])
        n = hi - lo
        if n == 0:
            continue
        picks = {0, n - 1, min(n - 1, 127), min(n - 1, 128)}
        if num_candidates is not None and num_candidates[u] > 0:
            h = n - int(num_candidates[u])
            picks |= {max(0, h - 1), min(n - 1, h), min(n - 1, h + 1)}
        picks |= set(rng.integers(0, n, size=per_user).tolist())
        rows += [lo + p for p in sorted(picks)]
    return np.array(rows, dtype=np.int64)
