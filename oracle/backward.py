"""Backward of the HSTU attention core, fp64 numpy (TEST INFRASTRUCTURE ONLY).

The forward (the C oracle, hstu_oracle.c) is, per user and head,
    s_ij = alpha q_i.k_j + rab_pos[p(i) - p(j) + N_max - 1] + rab_ts[b(i, j)]
    a_ij = SiLU(s_ij) / N_max on the allowed set M, else 0
    o_i  = sum_j a_ij v_j
("Generative Recommenders at Scale", Inside NVIDIA's GPU-native stack: SiLU
weighting with relative attention bias; training context in "How Generative
Recommenders Are Redefining RecSys at Scale").  With g = dL/do the chain rule
gives, on M (and zero elsewhere):
    dv_j      = sum_i a_ij g_i
    da_ij     = g_i . v_j
    ds_ij     = da_ij SiLU'(s_ij) / N_max,   SiLU'(x) = sig(x) (1 + x (1 - sig(x)))
    dq_i      = alpha sum_j ds_ij k_j
    dk_j      = alpha sum_i ds_ij q_i
    d rab_pos[p(i) - p(j) + N_max - 1] += ds_ij,   d rab_ts[b(i, j)] += ds_ij
Dense per-user matrices: for small inputs only.  Timestamps only select
buckets, so they get no gradient.
"""
from __future__ import annotations

import numpy as np

from . import _f64, _i32, _i64, ts_bucket


def attn_jagged_bwd(q, k, v, seq_offsets, timestamps, num_candidates, rab_pos, rab_ts, alpha: float,
                    n_max: int, d_o):
    """Returns dq, dk, dv [T, H, d] and d_rab_pos [2 n_max - 1], d_rab_ts [NB] (fp64)."""
    qd, kd, vd, g = _f64(q), _f64(k), _f64(v), _f64(d_o)
    T, H, d = qd.shape
    off = _i32(seq_offsets)
    ts = _i64(timestamps)
    cand = _i32(num_candidates)
    rp, rt = _f64(rab_pos), _f64(rab_ts)
    nb = len(rt)
    dq, dk, dv = np.zeros_like(qd), np.zeros_like(kd), np.zeros_like(vd)
    drp, drt = np.zeros_like(rp), np.zeros_like(rt)
    for u in range(len(off) - 1):
        lo, hi = int(off[u]), int(off[u + 1])
        n = hi - lo
        if n == 0:
            continue
        h = n - (int(cand[u]) if cand is not None else 0)
        idx = np.arange(n)
        pos = np.minimum(idx, h)
        ii, jj = np.meshgrid(idx, idx, indexing="ij")
        allowed = np.where(ii < h, jj <= ii, (jj < h) | (jj == ii))
        ridx = pos[:, None] - pos[None, :] + n_max - 1
        t = ts[lo:hi]
        bucket = ts_bucket((t[:, None] - t[None, :]).ravel(), nb).reshape(n, n)
        bias = rp[ridx] + rt[bucket]
        for hh in range(H):
            Q, K, V, G = qd[lo:hi, hh], kd[lo:hi, hh], vd[lo:hi, hh], g[lo:hi, hh]
            S = alpha * Q @ K.T + bias
            sig = 1.0 / (1.0 + np.exp(-S))
            A = np.where(allowed, S * sig / n_max, 0.0)
            dA = G @ V.T
            dS = np.where(allowed, dA * sig * (1.0 + S * (1.0 - sig)) / n_max, 0.0)
            dv[lo:hi, hh] = A.T @ G
            dq[lo:hi, hh] = alpha * dS @ K
            dk[lo:hi, hh] = alpha * dS.T @ Q
            np.add.at(drp, ridx[allowed], dS[allowed])
            np.add.at(drt, bucket[allowed], dS[allowed])
    return dq, dk, dv, drp, drt
