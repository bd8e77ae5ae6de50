"""Seeded synthetic inputs for HSTU jagged attention workloads.

This module only draws random numbers and lays them out; it computes nothing
of the attention method itself.  Both the CPU oracle (through the tests) and
the CUDA path (through the tests and the bench) take their inputs from here,
so the two sides see bit-identical values.

Workloads (shapes and distributions follow the workload descriptions that
accompany the HSTU pages, "Deploying an HSTU Generative Recommender" and
"HSTU Generative Recommenders: Deploy on GPU Cloud", M-FALCON section):

  tiny_fp32      2 users, lengths {37, 64}, 2 heads, d=32, fp32, N_max=64
  layer_bf16     32 users, lengths U{512..1024}, 4 heads, d=128, N_max=1024
  stack8_bf16    8 users, lengths U{4160..8320}, 4 heads, d=128, N_max=8320, 8 layers
  stack8_n8192   as stack8_bf16 but every length is 8192 (unmasked-tile target case)
  mfalcon_bf16   16 users, history U{2048..4096} + 512 candidates, N_max=4608, 2 layers
  paged_bf16     8 users, cached prefix U{6144..8192} in 32-token pages, +64 actions
                 +64 candidates, N_max=8320, 8 layers (one pool per layer)

Draw order inside one workload/layer: lengths, timestamps, rab tables,
weights, then X or Q/K/V/U.  Seeds are 1000 + workload id, and every layer
draws from its own stream ``default_rng([seed, layer])``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

WORKLOADS = {
    "tiny_fp32": 0,
    "layer_bf16": 1,
    "stack8_bf16": 2,
    "mfalcon_bf16": 3,
    "paged_bf16": 4,
    "stack8_n8192": 5,
}

NUM_TS_BUCKETS = 128
T0_BASE = 1_700_000_000  # seconds; large absolute values exercise 64-bit time arithmetic


@dataclasses.dataclass
class JaggedBatch:
    """One jagged attention problem, all arrays on the host.

    q, k, v: [T, H, d]; u: [T, H*d]; dtype torch.float32 or torch.bfloat16.
    seq_offsets: int32 [B+1]; timestamps: int64 [T]; num_candidates: int32 [B] or None.
    rab_pos: float32 [2*n_max-1]; rab_ts: float32 [num_ts_buckets].
    """
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    u: torch.Tensor
    seq_offsets: np.ndarray
    timestamps: np.ndarray
    num_candidates: Optional[np.ndarray]
    rab_pos: np.ndarray
    rab_ts: np.ndarray
    alpha: float
    n_max: int
    num_heads: int
    head_dim: int
    ln_gamma: Optional[np.ndarray] = None
    ln_beta: Optional[np.ndarray] = None
    ln_eps: float = 1e-5

    @property
    def batch(self) -> int:
        return len(self.seq_offsets) - 1

    @property
    def total_tokens(self) -> int:
        return int(self.seq_offsets[-1])

    @property
    def lengths(self) -> np.ndarray:
        return np.diff(self.seq_offsets)

    @property
    def max_seq_len(self) -> int:
        return int(self.lengths.max()) if self.batch else 0


@dataclasses.dataclass
class PagedBatch:
    """New tokens of each user plus a K/V prefix held in a paged pool.

    q, k, v: [T_new, H, d]; u: [T_new, H*d] (new tokens, jagged by new_offsets).
    k_pool, v_pool: [num_pages, H, page_size, d]; slots past a user's cached
    length hold NaN so that any read of them shows up in the output.
    kv_page_table: int32 [B, max_pages_per_user], -1 where unused.
    cached_lens: int32 [B]; timestamps: int64 jagged over prefix+new by ts_offsets.
    num_candidates: int32 [B]; candidates are the last new tokens of each user.
    """
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    u: torch.Tensor
    new_offsets: np.ndarray
    timestamps: np.ndarray
    ts_offsets: np.ndarray
    num_candidates: np.ndarray
    rab_pos: np.ndarray
    rab_ts: np.ndarray
    k_pool: torch.Tensor
    v_pool: torch.Tensor
    kv_page_table: np.ndarray
    cached_lens: np.ndarray
    page_size: int
    alpha: float
    n_max: int
    num_heads: int
    head_dim: int
    # the prefix K/V of every user, unpaged, for building the full-recompute reference
    k_prefix: list = dataclasses.field(default_factory=list)
    v_prefix: list = dataclasses.field(default_factory=list)
    ln_gamma: Optional[np.ndarray] = None
    ln_beta: Optional[np.ndarray] = None
    ln_eps: float = 1e-5

    @property
    def batch(self) -> int:
        return len(self.new_offsets) - 1


# ----------------------------------------------------------------------------
# primitive draws
# ----------------------------------------------------------------------------

def offsets_from_lengths(lengths) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    off = np.zeros(len(lengths) + 1, dtype=np.int64)
    np.cumsum(lengths, out=off[1:])
    return off.astype(np.int32)


def draw_timestamps(rng: np.random.Generator, history_lens, cand_lens=None,
                    mean_gap: float = 600.0) -> np.ndarray:
    """Non-decreasing int64 seconds per user: exponential gaps (rounded, at
    least 1 s) for history tokens; candidates repeat the last history time."""
    history_lens = np.asarray(history_lens, dtype=np.int64)
    if cand_lens is None:
        cand_lens = np.zeros_like(history_lens)
    out = []
    for h, c in zip(history_lens, np.asarray(cand_lens, dtype=np.int64)):
        t0 = T0_BASE + int(rng.integers(0, 1_000_000))
        gaps = np.maximum(1, np.rint(rng.exponential(mean_gap, size=max(int(h) - 1, 0)))).astype(np.int64)
        hist = t0 + np.concatenate([np.zeros(1 if h > 0 else 0, np.int64), np.cumsum(gaps)])
        last = hist[-1] if h > 0 else t0
        out.append(np.concatenate([hist, np.full(int(c), last, dtype=np.int64)]))
    return np.concatenate(out) if out else np.zeros(0, np.int64)


def draw_rab(rng: np.random.Generator, n_max: int, num_buckets: int = NUM_TS_BUCKETS,
             std: float = 0.02):
    rab_pos = rng.normal(0.0, std, size=2 * n_max - 1).astype(np.float32)
    rab_ts = rng.normal(0.0, std, size=num_buckets).astype(np.float32)
    return rab_pos, rab_ts


def draw_normal(rng: np.random.Generator, shape, scale: float, dtype: torch.dtype) -> torch.Tensor:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        a *= np.float32(scale)
    t = torch.from_numpy(a)
    return t if dtype == torch.float32 else t.to(dtype)


def xavier_uniform(rng: np.random.Generator, fan_in: int, fan_out: int) -> np.ndarray:
    bound = math.sqrt(6.0 / (fan_in + fan_out))
    return rng.uniform(-bound, bound, size=(fan_in, fan_out)).astype(np.float32)


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

def _rng(workload: str, layer: int = 0, seed: Optional[int] = None) -> np.random.Generator:
    base = 1000 + WORKLOADS[workload] if seed is None else seed
    return np.random.default_rng([base, layer])


def jagged_batch(lengths, num_heads: int, head_dim: int, n_max: int, *,
                 rng: np.random.Generator, dtype: torch.dtype = torch.bfloat16,
                 num_candidates=None, qkvu_scale: float = 1.0,
                 alpha: Optional[float] = None, rab_std: float = 0.02,
                 num_buckets: int = NUM_TS_BUCKETS, mean_gap: float = 600.0) -> JaggedBatch:
    """Generic jagged problem: draws timestamps, rab tables and Q/K/V/U."""
    lengths = np.asarray(lengths, dtype=np.int64)
    cand = None if num_candidates is None else np.asarray(num_candidates, dtype=np.int64)
    hist = lengths if cand is None else lengths - cand
    ts = draw_timestamps(rng, hist, cand, mean_gap)
    rab_pos, rab_ts = draw_rab(rng, n_max, num_buckets, rab_std)
    T = int(lengths.sum())
    H, d = num_heads, head_dim
    q = draw_normal(rng, (T, H, d), qkvu_scale, dtype)
    k = draw_normal(rng, (T, H, d), qkvu_scale, dtype)
    v = draw_normal(rng, (T, H, d), qkvu_scale, dtype)
    u = draw_normal(rng, (T, H * d), qkvu_scale, dtype)
    return JaggedBatch(q=q, k=k, v=v, u=u, seq_offsets=offsets_from_lengths(lengths),
                       timestamps=ts,
                       num_candidates=None if cand is None else cand.astype(np.int32),
                       rab_pos=rab_pos, rab_ts=rab_ts,
                       alpha=(1.0 / math.sqrt(d)) if alpha is None else alpha,
                       n_max=n_max, num_heads=H, head_dim=d)


def workload_attention(workload: str, layer: int = 0, seed: Optional[int] = None) -> JaggedBatch:
    """Attention-level inputs of a named workload (one layer)."""
    rng = _rng(workload, layer, seed)
    if workload == "tiny_fp32":
        return jagged_batch([37, 64], 2, 32, 64, rng=rng, dtype=torch.float32,
                            qkvu_scale=1.0 / math.sqrt(32))
    if workload == "layer_bf16":
        lengths = rng.integers(512, 1024, size=32, endpoint=True)
        return jagged_batch(lengths, 4, 128, 1024, rng=rng)
    if workload == "stack8_bf16":
        lengths = rng.integers(4160, 8320, size=8, endpoint=True)
        return jagged_batch(lengths, 4, 128, 8320, rng=rng)
    if workload == "stack8_n8192":
        return jagged_batch(np.full(8, 8192), 4, 128, 8320, rng=rng)
    if workload == "mfalcon_bf16":
        hist = rng.integers(2048, 4096, size=16, endpoint=True)
        return jagged_batch(hist + 512, 4, 128, 4608, rng=rng,
                            num_candidates=np.full(16, 512))
    raise ValueError(f"no jagged attention inputs for workload {workload!r}")


def paged_batch(cached_lens, num_actions, num_cands, num_heads: int, head_dim: int,
                n_max: int, *, rng: np.random.Generator, page_size: int = 32,
                dtype: torch.dtype = torch.bfloat16, qkvu_scale: float = 1.0,
                spare_pages: int = 7, poison: bool = True,
                num_buckets: int = NUM_TS_BUCKETS) -> PagedBatch:
    """Paged problem: prefix K/V scattered over a pool through a random page table."""
    cached = np.asarray(cached_lens, dtype=np.int64)
    B = len(cached)
    acts = np.broadcast_to(np.asarray(num_actions, dtype=np.int64), (B,)).copy()
    cands = np.broadcast_to(np.asarray(num_cands, dtype=np.int64), (B,)).copy()
    n_new = acts + cands
    ts = draw_timestamps(rng, cached + acts, cands)
    rab_pos, rab_ts = draw_rab(rng, n_max, num_buckets)
    H, d = num_heads, head_dim
    pages_per_user = (cached + page_size - 1) // page_size
    total_pages = int(pages_per_user.sum()) + spare_pages
    max_pages = max(1, int(pages_per_user.max()) if B else 1)
    perm = rng.permutation(total_pages)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    pos = 0
    for b in range(B):
        table[b, :pages_per_user[b]] = perm[pos:pos + pages_per_user[b]]
        pos += pages_per_user[b]
    fill = float("nan") if poison else 0.0
    k_pool = torch.full((total_pages, H, page_size, d), fill, dtype=torch.float32)
    v_pool = torch.full((total_pages, H, page_size, d), fill, dtype=torch.float32)
    k_prefix, v_prefix = [], []
    for b in range(B):
        L = int(cached[b])
        kp = draw_normal(rng, (L, H, d), qkvu_scale, dtype)
        vp = draw_normal(rng, (L, H, d), qkvu_scale, dtype)
        k_prefix.append(kp)
        v_prefix.append(vp)
        for pg in range(int(pages_per_user[b])):
            lo, hi = pg * page_size, min(L, (pg + 1) * page_size)
            phys = int(table[b, pg])
            k_pool[phys, :, : hi - lo, :] = kp[lo:hi].float().permute(1, 0, 2)
            v_pool[phys, :, : hi - lo, :] = vp[lo:hi].float().permute(1, 0, 2)
    T_new = int(n_new.sum())
    q = draw_normal(rng, (T_new, H, d), qkvu_scale, dtype)
    k = draw_normal(rng, (T_new, H, d), qkvu_scale, dtype)
    v = draw_normal(rng, (T_new, H, d), qkvu_scale, dtype)
    u = draw_normal(rng, (T_new, H * d), qkvu_scale, dtype)
    return PagedBatch(q=q, k=k, v=v, u=u, new_offsets=offsets_from_lengths(n_new),
                      timestamps=ts, ts_offsets=offsets_from_lengths(cached + n_new),
                      num_candidates=cands.astype(np.int32), rab_pos=rab_pos, rab_ts=rab_ts,
                      k_pool=k_pool.to(dtype), v_pool=v_pool.to(dtype), kv_page_table=table,
                      cached_lens=cached.astype(np.int32), page_size=page_size,
                      alpha=1.0 / math.sqrt(d), n_max=n_max, num_heads=H, head_dim=d,
                      k_prefix=k_prefix, v_prefix=v_prefix)


def workload_paged(layer: int = 0, seed: Optional[int] = None) -> PagedBatch:
    rng = _rng("paged_bf16", layer, seed)
    cached = rng.integers(6144, 8192, size=8, endpoint=True)
    return paged_batch(cached, 64, 64, 4, 128, 8320, rng=rng)


@dataclasses.dataclass
class LayerWeights:
    w1: np.ndarray  # [d_model, 4*H*d]  columns ordered [U | V | Q | K], head-major in each block
    b1: np.ndarray  # [4*H*d]
    w2: np.ndarray  # [H*d, d_model]
    b2: np.ndarray  # [d_model]


def layer_weights(rng: np.random.Generator, d_model: int, num_heads: int, head_dim: int) -> LayerWeights:
    hd = num_heads * head_dim
    return LayerWeights(w1=xavier_uniform(rng, d_model, 4 * hd), b1=np.zeros(4 * hd, np.float32),
                        w2=xavier_uniform(rng, hd, d_model), b2=np.zeros(d_model, np.float32))


@dataclasses.dataclass
class StackInputs:
    x: torch.Tensor                 # [T, d_model] bf16
    seq_offsets: np.ndarray
    timestamps: np.ndarray
    num_candidates: Optional[np.ndarray]
    layers: list                    # per layer: (rab_pos, rab_ts, LayerWeights)
    n_max: int
    num_heads: int
    head_dim: int
    d_model: int
    alpha: float


def workload_stack(workload: str, num_layers: Optional[int] = None,
                   seed: Optional[int] = None) -> StackInputs:
    """Inputs of a layer stack: X plus per-layer rab tables and weights."""
    rng = _rng(workload, 0, seed)
    cand = None
    if workload == "layer_bf16":
        lengths, n_max, L = rng.integers(512, 1024, size=32, endpoint=True), 1024, 1
    elif workload == "stack8_bf16":
        lengths, n_max, L = rng.integers(4160, 8320, size=8, endpoint=True), 8320, 8
    elif workload == "mfalcon_bf16":
        hist = rng.integers(2048, 4096, size=16, endpoint=True)
        cand = np.full(16, 512)
        lengths, n_max, L = hist + 512, 4608, 2
    else:
        raise ValueError(f"no layer-stack inputs for workload {workload!r}")
    L = L if num_layers is None else num_layers
    hist = lengths if cand is None else lengths - cand
    ts = draw_timestamps(rng, hist, cand)
    H, d, dm = 4, 128, 512
    rabs = [draw_rab(rng, n_max) for _ in range(L)]
    weights = [layer_weights(rng, dm, H, d) for _ in range(L)]
    T = int(np.sum(lengths))
    x = draw_normal(rng, (T, dm), 1.0, torch.bfloat16)
    return StackInputs(x=x, seq_offsets=offsets_from_lengths(lengths), timestamps=ts,
                       num_candidates=None if cand is None else cand.astype(np.int32),
                       layers=[(rp, rt, w) for (rp, rt), w in zip(rabs, weights)],
                       n_max=n_max, num_heads=H, head_dim=d, d_model=dm, alpha=1.0 / math.sqrt(d))


def attention_stack(workload: str, num_layers: Optional[int] = None, seed: Optional[int] = None):
    """Attention inputs of every layer of a stack: one set of users, lengths and
    timestamps (drawn from the layer-0 stream), per-layer rab tables and
    Q/K/V/U (drawn from each layer's own stream)."""
    base = workload_attention(workload, layer=0, seed=seed)
    layers = {"stack8_bf16": 8, "stack8_n8192": 8, "mfalcon_bf16": 2, "layer_bf16": 1, "tiny_fp32": 1}
    L = layers[workload] if num_layers is None else num_layers
    out = [base]
    T, H, d = base.q.shape
    for layer in range(1, L):
        rng = _rng(workload, layer, seed)
        rab_pos, rab_ts = draw_rab(rng, base.n_max)
        q = draw_normal(rng, (T, H, d), 1.0, base.q.dtype)
        k = draw_normal(rng, (T, H, d), 1.0, base.q.dtype)
        v = draw_normal(rng, (T, H, d), 1.0, base.q.dtype)
        u = draw_normal(rng, (T, H * d), 1.0, base.q.dtype)
        out.append(dataclasses.replace(base, q=q, k=k, v=v, u=u, rab_pos=rab_pos, rab_ts=rab_ts))
    return out


def paged_stack(num_layers: int = 8, seed: Optional[int] = None):
    """The paged workload of every layer: one set of users and cached lengths,
    a separate page pool and page table per layer."""
    rng0 = _rng("paged_bf16", 0, seed)
    cached = rng0.integers(6144, 8192, size=8, endpoint=True)
    out = []
    for layer in range(num_layers):
        rng = _rng("paged_bf16", 100 + layer, seed)
        out.append(paged_batch(cached, 64, 64, 4, 128, 8320, rng=rng))
    return out
