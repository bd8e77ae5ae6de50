"""Pins of the backward oracle (oracle/backward.py) by central finite
differences of the forward C oracle's raw A.V output: for L = sum(g * o), the
directional derivative along random directions of q, k, v, rab_pos and rab_ts
must match the analytic gradients.  The forward oracle is pinned on its own
(test_oracle.py), and the two share no arithmetic."""
import numpy as np
import pytest

import oracle
from oracle import backward as obwd


def problem(lengths, cands, H=2, d=4, n_max=16, seed=0):
    rng = np.random.default_rng(seed)
    T = int(sum(lengths))
    q, k, v = (rng.standard_normal((T, H, d)) for _ in range(3))
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    ts = []
    for n, c in zip(lengths, cands):
        t = 1_700_000_000 + np.cumsum(rng.integers(1, 2000, size=n))
        if c:
            t[n - c:] = t[n - c - 1]
        ts.append(t)
    ts = np.concatenate(ts).astype(np.int64)
    rp = rng.standard_normal(2 * n_max - 1) * 0.3
    rt = rng.standard_normal(128) * 0.3
    g = rng.standard_normal((T, H, d))
    return dict(q=q, k=k, v=v, off=off, ts=ts, cand=np.array(cands, np.int32), rp=rp, rt=rt, g=g, n_max=n_max,
                alpha=0.7)


def loss(P, **over):
    x = dict(P, **over)
    T, H, d = x["q"].shape
    _, o = oracle.attn_jagged(x["q"], x["k"], x["v"], np.ones((T, H * d)), x["off"], x["ts"], x["cand"], x["rp"],
                              x["rt"], x["alpha"], x["n_max"], want_o=True)
    return float(np.sum(x["g"] * o))


@pytest.mark.parametrize("lengths,cands", [([6, 4], [0, 0]), ([7, 5], [2, 0]), ([1, 9], [0, 4])])
def test_gradients_match_finite_differences(lengths, cands):
    P = problem(lengths, cands, seed=sum(lengths) + sum(cands))
    dq, dk, dv, drp, drt = obwd.attn_jagged_bwd(P["q"], P["k"], P["v"], P["off"], P["ts"], P["cand"], P["rp"],
                                                 P["rt"], P["alpha"], P["n_max"], P["g"])
    rng = np.random.default_rng(5)
    eps = 1e-5
    for name, grad in (("q", dq), ("k", dk), ("v", dv), ("rp", drp), ("rt", drt)):
        for _ in range(3):
            delta = rng.standard_normal(P[name].shape)
            fd = (loss(P, **{name: P[name] + eps * delta}) - loss(P, **{name: P[name] - eps * delta})) / (2 * eps)
            an = float(np.sum(grad * delta))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_single_entries_of_the_bias_tables():
    P = problem([8, 3], [3, 0], seed=11)
    _, _, _, drp, drt = obwd.attn_jagged_bwd(P["q"], P["k"], P["v"], P["off"], P["ts"], P["cand"], P["rp"],
                                             P["rt"], P["alpha"], P["n_max"], P["g"])
    eps = 1e-6
    for name, grad in (("rp", drp), ("rt", drt)):
        for idx in np.nonzero(grad)[0][:6]:
            e = np.zeros_like(P[name])
            e[idx] = eps
            fd = (loss(P, **{name: P[name] + e}) - loss(P, **{name: P[name] - e})) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(grad[idx]))
    # entries no allowed pair indexes get no gradient
    assert np.all(drp[:P["n_max"] - 8] == 0.0)         # p(i) - p(j) >= -(n-1) never used on the causal side
