"""HSTU layer glue around the attention, fp64 numpy (TEST INFRASTRUCTURE ONLY).

Source: "How Generative Recommenders Are Redefining RecSys at Scale"
(Takeaways): gating is applied before the output projection; the layer's
input projection produces U, V, Q, K through SiLU.  Readings (the pages give
no formula): f1 is one linear map d_model -> 4*H*d followed by SiLU whose
output columns are ordered [U | V | Q | K], head-major inside each block; f2
is a linear map H*d -> d_model; there is no residual and no input norm.
"""
from __future__ import annotations

import numpy as np

from . import attn_jagged


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def f1(x, w1, b1, num_heads: int, head_dim: int):
    """[U | V | Q | K] = SiLU(x W1 + b1); returns u [T,H*d], v,q,k [T,H,d]."""
    x = np.asarray(x, np.float64)
    z = silu(x @ np.asarray(w1, np.float64) + np.asarray(b1, np.float64))
    hd = num_heads * head_dim
    T = x.shape[0]
    u = z[:, 0 * hd:1 * hd]
    v = z[:, 1 * hd:2 * hd].reshape(T, num_heads, head_dim)
    q = z[:, 2 * hd:3 * hd].reshape(T, num_heads, head_dim)
    k = z[:, 3 * hd:4 * hd].reshape(T, num_heads, head_dim)
    return u, v, q, k


def f2(y, w2, b2):
    return np.asarray(y, np.float64) @ np.asarray(w2, np.float64) + np.asarray(b2, np.float64)


def layer(x, w1, b1, w2, b2, seq_offsets, timestamps, num_candidates, rab_pos, rab_ts,
          alpha: float, n_max: int, num_heads: int, head_dim: int, rows=None):
    """One HSTU layer: x -> f1 -> attention (LayerNorm(A V) * U) -> f2.

    rows: optional subset of output rows (attention is evaluated only there)."""
    u, v, q, k = f1(x, w1, b1, num_heads, head_dim)
    y = attn_jagged(q, k, v, u, seq_offsets, timestamps, num_candidates, rab_pos, rab_ts,
                    alpha, n_max, rows=rows)
    return f2(y, w2, b2)
