"""fp64 CPU oracle for HSTU jagged attention (TEST INFRASTRUCTURE ONLY).

Only tests/, the smoke check in __graft_entry__ and the bench's CPU-baseline
leg may import this package.  It shares no code with the CUDA library:
the attention itself is plain C in ``hstu_oracle.c`` (fp64, loops over the
allowed set, OpenMP over query rows), wrapped here with ctypes; the layer glue
around it is plain numpy fp64 in ``layer.py``.

Every function follows the definition written at the top of hstu_oracle.c.
Pins: the bucket is pinned to an exact decimal evaluation, the attention to
closed forms, one-hot bias probes, brute-force loops on tiny inputs and the
method's invariants (tests/test_oracle.py).  Parity is not pinned to the
pages themselves: they print no worked example or intermediate value.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hstu_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (fp64, -O2, OpenMP, libquadmath)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math", "-std=gnu11",
               "-o", tmp, _SRC, "-lquadmath", "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.oracle_ts_bucket.argtypes = [i64, i32]
        lib.oracle_ts_bucket.restype = i32
        lib.oracle_ts_bucket_array.argtypes = [P, i64, i32, P]
        lib.oracle_ts_bucket_array.restype = None
        lib.oracle_attn_jagged.argtypes = [P, P, P, P, P, i32, P, P, P, P, i32, f64, i32, i32, i32,
                                           P, P, f64, P, i64, P, P]
        lib.oracle_attn_jagged.restype = ctypes.c_int
        lib.oracle_attn_paged.argtypes = [P, P, P, P, P, i32, P, P, P, P, P, i32, f64, i32, i32,
                                          i32, P, P, f64, P, P, P, i32, i32, P, P, i64, P, P]
        lib.oracle_attn_paged.restype = ctypes.c_int
        lib.oracle_allowed_pairs.argtypes = [P, i32, P]
        lib.oracle_allowed_pairs.restype = i64
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor (any float dtype): exact upcast
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a) -> Optional[np.ndarray]:
    return None if a is None else np.ascontiguousarray(a, dtype=np.int32)


def _i64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int64)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n else len(os.sched_getaffinity(0))


def ts_bucket(dt, num_buckets: int = 128) -> np.ndarray:
    """clamp(floor(ln(|dt|+1)/0.301), 0, num_buckets-1), elementwise, exact."""
    dt = _i64(np.atleast_1d(dt))
    out = np.empty(dt.shape, dtype=np.int32)
    _load().oracle_ts_bucket_array(_ptr(dt), dt.size, num_buckets, _ptr(out))
    return out


def attn_jagged(q, k, v, u, seq_offsets, timestamps, num_candidates, rab_pos, rab_ts,
                alpha: float, n_max: int, gamma=None, beta=None, eps: float = 1e-5,
                rows: Optional[Sequence[int]] = None, want_o: bool = False):
    """y [R, H*d] (and o [R, H, d] if want_o) for every row, or the given rows."""
    qd, kd, vd, ud = _f64(q), _f64(k), _f64(v), _f64(u)
    T, H, d = qd.shape
    off = _i32(seq_offsets)
    B = len(off) - 1
    ts = _i64(timestamps)
    cand = _i32(num_candidates)
    rp, rt = _f64(rab_pos), _f64(rab_ts)
    g = None if gamma is None else _f64(gamma)
    b_ = None if beta is None else _f64(beta)
    rr = None if rows is None else _i64(rows)
    R = T if rr is None else len(rr)
    y = np.empty((R, H * d), np.float64)
    o = np.empty((R, H, d), np.float64) if want_o else None
    rc = _load().oracle_attn_jagged(_ptr(qd), _ptr(kd), _ptr(vd), _ptr(ud), _ptr(off), B, _ptr(ts),
                                    _ptr(cand), _ptr(rp), _ptr(rt), len(rt), float(alpha), int(n_max),
                                    H, d, _ptr(g), _ptr(b_), float(eps), _ptr(rr), R, _ptr(o), _ptr(y))
    if rc != 0:
        raise ValueError("oracle_attn_jagged: bad argument")
    return (y, o) if want_o else y


def attn_paged(q, k, v, u, new_offsets, timestamps, ts_offsets, num_candidates, rab_pos, rab_ts,
               alpha: float, n_max: int, k_pool, v_pool, page_table, page_size: int, cached_lens,
               gamma=None, beta=None, eps: float = 1e-5, rows: Optional[Sequence[int]] = None,
               want_o: bool = False):
    qd, kd, vd, ud = _f64(q), _f64(k), _f64(v), _f64(u)
    T, H, d = qd.shape
    off = _i32(new_offsets)
    B = len(off) - 1
    ts, tso = _i64(timestamps), _i32(ts_offsets)
    cand = _i32(num_candidates)
    rp, rt = _f64(rab_pos), _f64(rab_ts)
    kp, vp = _f64(k_pool), _f64(v_pool)
    pt = _i32(page_table)
    cl = _i32(cached_lens)
    g = None if gamma is None else _f64(gamma)
    b_ = None if beta is None else _f64(beta)
    rr = None if rows is None else _i64(rows)
    R = T if rr is None else len(rr)
    y = np.empty((R, H * d), np.float64)
    o = np.empty((R, H, d), np.float64) if want_o else None
    rc = _load().oracle_attn_paged(_ptr(qd), _ptr(kd), _ptr(vd), _ptr(ud), _ptr(off), B, _ptr(ts),
                                   _ptr(tso), _ptr(cand), _ptr(rp), _ptr(rt), len(rt), float(alpha),
                                   int(n_max), H, d, _ptr(g), _ptr(b_), float(eps), _ptr(kp), _ptr(vp),
                                   _ptr(pt), pt.shape[1], int(page_size), _ptr(cl), _ptr(rr), R,
                                   _ptr(o), _ptr(y))
    if rc != 0:
        raise ValueError("oracle_attn_paged: bad argument")
    return (y, o) if want_o else y


def allowed_pairs(seq_offsets, num_candidates=None) -> int:
    off = _i32(seq_offsets)
    cand = _i32(num_candidates)
    return int(_load().oracle_allowed_pairs(_ptr(off), len(off) - 1, _ptr(cand)))


def batch_attn(batch, rows=None, want_o: bool = False):
    """Oracle on a synth.JaggedBatch."""
    return attn_jagged(batch.q, batch.k, batch.v, batch.u, batch.seq_offsets, batch.timestamps,
                       batch.num_candidates, batch.rab_pos, batch.rab_ts, batch.alpha, batch.n_max,
                       batch.ln_gamma, batch.ln_beta, batch.ln_eps, rows=rows, want_o=want_o)


def batch_paged(pb, rows=None, want_o: bool = False):
    """Oracle on a synth.PagedBatch."""
    return attn_paged(pb.q, pb.k, pb.v, pb.u, pb.new_offsets, pb.timestamps, pb.ts_offsets,
                      pb.num_candidates, pb.rab_pos, pb.rab_ts, pb.alpha, pb.n_max, pb.k_pool,
                      pb.v_pool, pb.kv_page_table, pb.page_size, pb.cached_lens, pb.ln_gamma,
                      pb.ln_beta, pb.ln_eps, rows=rows, want_o=want_o)
