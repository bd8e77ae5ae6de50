"""Python entry points over libhstu.so, with the same names as the C ABI.

Tensors are torch CUDA tensors (torch provides device memory and the current
stream); everything else is the library's.  Inputs on the CPU are refused.
"""
from __future__ import annotations

import ctypes
import math
from typing import Optional

import torch

from . import _lib

_DT = {torch.float32: _lib.DT_F32, torch.bfloat16: _lib.DT_BF16}


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream] = None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(name: str, t: Optional[torch.Tensor], dtype=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _rows_view(name: str, t: torch.Tensor, H: int, d: int) -> int:
    """Token stride (elements) of a [T,H,d] (or [T,H*d]) view with packed heads."""
    if t.numel() == 0:
        return H * d  # no rows: the layout is immaterial
    if t.dim() == 3:
        ok = t.stride(2) == 1 and t.stride(1) == d
    else:
        ok = t.stride(1) == 1
    if not ok:
        raise ValueError(f"{name}: heads and features must be packed (stride 1 / d)")
    return t.stride(0) if t.shape[0] > 1 else H * d


def attn_params(*, batch: int, num_heads: int, head_dim: int, n_max: int, total_tokens: int,
                max_seq_len: int, dtype: torch.dtype, alpha: Optional[float] = None,
                num_ts_buckets: int = 128, qkv_stride: int = 0, u_stride: int = 0,
                ln_eps: float = 1e-5, flags: int = 0) -> _lib.AttnParams:
    return _lib.AttnParams(batch=batch, num_heads=num_heads, head_dim=head_dim, n_max=n_max,
                           num_ts_buckets=num_ts_buckets, total_tokens=total_tokens,
                           max_seq_len=max_seq_len, qkv_stride=qkv_stride, u_stride=u_stride,
                           alpha=(1.0 / math.sqrt(head_dim)) if alpha is None else alpha,
                           ln_eps=ln_eps, dtype=_DT[dtype], flags=flags)


def hstu_attn_workspace_size(p: _lib.AttnParams) -> int:
    return int(_lib.load().hstu_attn_workspace_size(ctypes.byref(p)))


def hstu_attn_paged_workspace_size(p: _lib.AttnParams, num_splits: int) -> int:
    return int(_lib.load().hstu_attn_paged_workspace_size(ctypes.byref(p), num_splits))


def hstu_attn_paged_default_splits(p: _lib.AttnParams, max_cached_len: int) -> int:
    return int(_lib.load().hstu_attn_paged_default_splits(ctypes.byref(p), max_cached_len))


def hstu_attn_fwd(q, k, v, u, seq_offsets, timestamps, rab_pos, rab_ts, *, n_max: int,
                  alpha: Optional[float] = None, num_candidates=None, ln_gamma=None, ln_beta=None,
                  ln_eps: float = 1e-5, max_seq_len: Optional[int] = None, out=None,
                  workspace=None, raw_av: bool = False, force_simt: bool = False, stages: int = 0,
                  stream=None, params: Optional[_lib.AttnParams] = None, precise_silu: bool = False):
    """Jagged HSTU attention forward; returns out [T, H*d] (or o [T,H,d] fp32 when raw_av)."""
    T, H, d = q.shape
    dt = q.dtype
    for name, t in (("q", q), ("k", k), ("v", v), ("u", u)):
        _need_cuda(name, t, dt)
    _need_cuda("seq_offsets", seq_offsets, torch.int32)
    _need_cuda("timestamps", timestamps, torch.int64)
    _need_cuda("num_candidates", num_candidates, torch.int32)
    for name, t in (("rab_pos", rab_pos), ("rab_ts", rab_ts), ("ln_gamma", ln_gamma), ("ln_beta", ln_beta)):
        _need_cuda(name, t, torch.float32)
    qs = _rows_view("q", q, H, d)
    if _rows_view("k", k, H, d) != qs or _rows_view("v", v, H, d) != qs:
        raise ValueError("q, k and v must share one token stride")
    us = _rows_view("u", u, H, d)
    B = seq_offsets.numel() - 1
    flags = ((_lib.F_OUTPUT_RAW_AV if raw_av else 0) | (_lib.F_FORCE_SIMT if force_simt else 0) |
             (_lib.F_PRECISE_SILU if precise_silu else 0) | stages)
    if params is None:
        params = attn_params(batch=B, num_heads=H, head_dim=d, n_max=n_max, total_tokens=T,
                             max_seq_len=n_max if max_seq_len is None else max_seq_len, dtype=dt,
                             alpha=alpha, num_ts_buckets=rab_ts.numel(), qkv_stride=qs, u_stride=us,
                             ln_eps=ln_eps, flags=flags)
    if out is None:
        out = (torch.empty(T, H, d, dtype=torch.float32, device=q.device) if raw_av
               else torch.empty(T, H * d, dtype=dt, device=q.device))
    if workspace is None:
        workspace = torch.empty(hstu_attn_workspace_size(params), dtype=torch.uint8, device=q.device)
    rc = _lib.load().hstu_attn_fwd(ctypes.byref(params), _p(q), _p(k), _p(v), _p(u), _p(seq_offsets),
                                   _p(timestamps), _p(num_candidates), _p(rab_pos), _p(rab_ts),
                                   _p(ln_gamma), _p(ln_beta), _p(out), _p(workspace),
                                   workspace.numel(), _stream(stream))
    _lib.check(rc, "hstu_attn_fwd")
    return out


def hstu_attn_fwd_paged(q, k, v, u, new_offsets, timestamps, ts_offsets, rab_pos, rab_ts, k_pool,
                        v_pool, kv_page_table, cached_lens, *, n_max: int, alpha: Optional[float] = None,
                        num_candidates=None, ln_gamma=None, ln_beta=None, ln_eps: float = 1e-5,
                        max_seq_len: Optional[int] = None, num_splits: Optional[int] = None,
                        max_cached_len: Optional[int] = None, out=None, workspace=None,
                        raw_av: bool = False, force_simt: bool = False, stages: int = 0, stream=None,
                        precise_silu: bool = False):
    """Incremental HSTU attention of new tokens over a paged K/V prefix."""
    T, H, d = q.shape
    dt = q.dtype
    for name, t in (("q", q), ("k", k), ("v", v), ("u", u), ("k_pool", k_pool), ("v_pool", v_pool)):
        _need_cuda(name, t, dt)
    for name, t in (("new_offsets", new_offsets), ("ts_offsets", ts_offsets),
                    ("kv_page_table", kv_page_table), ("cached_lens", cached_lens),
                    ("num_candidates", num_candidates)):
        _need_cuda(name, t, torch.int32)
    _need_cuda("timestamps", timestamps, torch.int64)
    if not (k_pool.is_contiguous() and v_pool.is_contiguous() and kv_page_table.is_contiguous()):
        raise ValueError("k_pool, v_pool and kv_page_table must be contiguous")
    num_pages, _, page_size, _ = k_pool.shape
    qs = _rows_view("q", q, H, d)
    if _rows_view("k", k, H, d) != qs or _rows_view("v", v, H, d) != qs:
        raise ValueError("q, k and v must share one token stride")
    us = _rows_view("u", u, H, d)
    B = new_offsets.numel() - 1
    flags = ((_lib.F_OUTPUT_RAW_AV if raw_av else 0) | (_lib.F_FORCE_SIMT if force_simt else 0) |
             (_lib.F_PRECISE_SILU if precise_silu else 0) | stages)
    params = attn_params(batch=B, num_heads=H, head_dim=d, n_max=n_max, total_tokens=T,
                         max_seq_len=n_max if max_seq_len is None else max_seq_len, dtype=dt,
                         alpha=alpha, num_ts_buckets=rab_ts.numel(), qkv_stride=qs, u_stride=us,
                         ln_eps=ln_eps, flags=flags)
    if num_splits is None:
        mc = n_max if max_cached_len is None else max_cached_len
        num_splits = hstu_attn_paged_default_splits(params, mc)
    if out is None:
        out = (torch.empty(T, H, d, dtype=torch.float32, device=q.device) if raw_av
               else torch.empty(T, H * d, dtype=dt, device=q.device))
    if workspace is None:
        workspace = torch.empty(hstu_attn_paged_workspace_size(params, num_splits), dtype=torch.uint8,
                                device=q.device)
    rc = _lib.load().hstu_attn_fwd_paged(
        ctypes.byref(params), _p(q), _p(k), _p(v), _p(u), _p(new_offsets), _p(timestamps), _p(ts_offsets),
        _p(num_candidates), _p(rab_pos), _p(rab_ts), _p(ln_gamma), _p(ln_beta), _p(k_pool), _p(v_pool),
        num_pages, _p(kv_page_table), kv_page_table.shape[1], page_size, _p(cached_lens), num_splits,
        _p(out), _p(workspace), workspace.numel(), _stream(stream))
    _lib.check(rc, "hstu_attn_fwd_paged")
    return out


def hstu_ts_bucket(dt: torch.Tensor, num_buckets: int = 128, out=None, stream=None) -> torch.Tensor:
    _need_cuda("dt", dt, torch.int64)
    dt = dt.contiguous()
    if out is None:
        out = torch.empty(dt.shape, dtype=torch.int32, device=dt.device)
    rc = _lib.load().hstu_ts_bucket(_p(dt), dt.numel(), num_buckets, _p(out), _stream(stream))
    _lib.check(rc, "hstu_ts_bucket")
    return out


def hstu_check_device_error(workspace: torch.Tensor, stream=None) -> int:
    """Synchronises the stream and returns the device status word of `workspace`."""
    return int(_lib.load().hstu_check_device_error(_p(workspace), _stream(stream)))


def hstu_status_string(status: int) -> str:
    return _lib.load().hstu_status_string(status).decode()


def hstu_version() -> int:
    return int(_lib.load().hstu_version())


def hstu_attn_fwd_static_ws(q, k, v, u, seq_offsets, timestamps, rab_pos, rab_ts, *, n_max: int,
                            alpha: Optional[float] = None, num_candidates=None, ln_gamma=None,
                            ln_beta=None, ln_eps: float = 1e-5, max_seq_len: Optional[int] = None,
                            out=None, stream=None):
    """hstu_attn_fwd without a workspace: the library's own 16 MiB device scratch is
    used instead (for callers that cannot allocate device memory where they run
    attention).  `out` may be given so that the call allocates nothing at all."""
    T, H, d = q.shape
    dt = q.dtype
    for name, t in (("q", q), ("k", k), ("v", v), ("u", u)):
        _need_cuda(name, t, dt)
    qs = _rows_view("q", q, H, d)
    us = _rows_view("u", u, H, d)
    params = attn_params(batch=seq_offsets.numel() - 1, num_heads=H, head_dim=d, n_max=n_max,
                         total_tokens=T, max_seq_len=n_max if max_seq_len is None else max_seq_len,
                         dtype=dt, alpha=alpha, num_ts_buckets=rab_ts.numel(), qkv_stride=qs,
                         u_stride=us, ln_eps=ln_eps)
    if out is None:
        out = torch.empty(T, H * d, dtype=dt, device=q.device)
    rc = _lib.load().hstu_attn_fwd_static_ws(ctypes.byref(params), _p(q), _p(k), _p(v), _p(u), _p(seq_offsets), _p(timestamps),
            _p(num_candidates), _p(rab_pos), _p(rab_ts), _p(ln_gamma), _p(ln_beta), _p(out),
            _stream(stream))
    _lib.check(rc, "hstu_attn_fwd_static_ws")
    return out


def linear_params(x: torch.Tensor, w: torch.Tensor, out: torch.Tensor, silu: bool,
                  force_cublas: bool = False) -> _lib.LinearParams:
    return _lib.LinearParams(rows=x.shape[0], d_in=x.shape[1], d_out=w.shape[1],
                             x_stride=x.stride(0) if x.shape[0] > 1 else x.shape[1],
                             out_stride=out.stride(0) if out.shape[0] > 1 else out.shape[1],
                             dtype=_DT[x.dtype],
                             flags=(_lib.LIN_SILU if silu else 0) | (_lib.LIN_CUBLAS if force_cublas else 0))


def hstu_linear_workspace_size(p: Optional[_lib.LinearParams] = None) -> int:
    p = p if p is not None else _lib.LinearParams()
    return int(_lib.load().hstu_linear_workspace_size(ctypes.byref(p)))


def _linear(name: str, x, w, bias, out, workspace, stream, silu: bool, force_cublas: bool = False):
    for nm, t in (("x", x), ("w", w), ("out", out)):
        _need_cuda(nm, t, x.dtype)
    _need_cuda("bias", bias, torch.float32)
    if x.dim() != 2 or w.dim() != 2 or x.shape[1] != w.shape[0]:
        raise ValueError(f"{name}: x [T, d_in] and w [d_in, d_out] expected")
    if x.stride(1) != 1 or not w.is_contiguous():
        raise ValueError(f"{name}: x rows and w must be contiguous")
    if out is None:
        out = torch.empty(x.shape[0], w.shape[1], dtype=x.dtype, device=x.device)
    if out.dim() != 2 or out.shape != (x.shape[0], w.shape[1]) or out.stride(1) != 1:
        raise ValueError(f"{name}: out [T, d_out] with contiguous rows expected")
    p = linear_params(x, w, out, silu, force_cublas)
    if workspace is None:
        workspace = torch.empty(hstu_linear_workspace_size(p), dtype=torch.uint8, device=x.device)
    rc = getattr(_lib.load(), name)(ctypes.byref(p), _p(x), _p(w), _p(bias), _p(out), _p(workspace),
                                    workspace.numel(), _stream(stream))
    _lib.check(rc, name)
    return out


def hstu_layer_f1(x, w1, b1=None, *, out=None, workspace=None, stream=None, force_cublas: bool = False):
    """[U | V | Q | K] = SiLU(x W1 + b1) as one [T, 4*H*d] tensor (blocks head-major)."""
    return _linear("hstu_layer_f1", x, w1, b1, out, workspace, stream, True, force_cublas)


def hstu_layer_f2(y, w2, b2=None, *, out=None, workspace=None, stream=None, force_cublas: bool = False):
    """x_next = y W2 + b2."""
    return _linear("hstu_layer_f2", y, w2, b2, out, workspace, stream, False, force_cublas)


def hstu_linear(x, w, bias=None, *, silu: bool = False, out=None, workspace=None, stream=None,
                force_cublas: bool = False):
    """out = act(x W + bias), act = SiLU or identity."""
    return _linear("hstu_linear", x, w, bias, out, workspace, stream, silu, force_cublas)


def split_uvqk(uvqk: torch.Tensor, num_heads: int, head_dim: int):
    """Views u [T, H*d] and v, q, k [T, H, d] of f1's [T, 4*H*d] output (no copy)."""
    hd = num_heads * head_dim
    T = uvqk.shape[0]
    u = uvqk[:, 0:hd]
    v, q, k = (uvqk[:, b * hd:(b + 1) * hd].unflatten(1, (num_heads, head_dim)) for b in (1, 2, 3))
    return u, v, q, k


def kv_params(k_pool: torch.Tensor, page_table: torch.Tensor, k_new: Optional[torch.Tensor] = None) -> _lib.KvParams:
    num_pages, H, P, d = k_pool.shape
    stride = 0 if k_new is None or k_new.shape[0] <= 1 else k_new.stride(0)
    return _lib.KvParams(batch=page_table.shape[0], num_heads=H, head_dim=d, page_size=P, num_pages=num_pages,
                         max_pages_per_user=page_table.shape[1], kv_stride=stride,
                         total_new=0 if k_new is None else k_new.shape[0], dtype=_DT[k_pool.dtype])


def hstu_kv_workspace_size(p: _lib.KvParams) -> int:
    return int(_lib.load().hstu_kv_workspace_size(ctypes.byref(p)))


def _kv_check(k_pool, page_table, cached_lens, free_pages, free_count):
    _need_cuda("k_pool", k_pool)
    for name, t in (("page_table", page_table), ("cached_lens", cached_lens), ("free_pages", free_pages),
                    ("free_count", free_count)):
        _need_cuda(name, t, torch.int32)
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if not k_pool.is_contiguous():
        raise ValueError("k_pool must be contiguous")


def hstu_kv_append(k_new, v_new, new_offsets, k_pool, v_pool, page_table, cached_lens, free_pages, free_count, *,
                   num_append=None, workspace=None, stream=None):
    """Appends the first num_append[u] new tokens of every user (all when None)
    behind its cached prefix, taking pages from the free stack; in place."""
    _kv_check(k_pool, page_table, cached_lens, free_pages, free_count)
    for name, t in (("k_new", k_new), ("v_new", v_new), ("v_pool", v_pool)):
        _need_cuda(name, t, k_pool.dtype)
    _need_cuda("new_offsets", new_offsets, torch.int32)
    _need_cuda("num_append", num_append, torch.int32)
    if k_new.stride() != v_new.stride() or k_new.stride(2) != 1 or k_new.stride(1) != k_new.shape[2]:
        raise ValueError("k_new and v_new must be [T, H, d] views with packed heads and one token stride")
    p = kv_params(k_pool, page_table, k_new)
    if workspace is None:
        workspace = torch.empty(hstu_kv_workspace_size(p), dtype=torch.uint8, device=k_pool.device)
    rc = _lib.load().hstu_kv_append(ctypes.byref(p), _p(k_new), _p(v_new), _p(new_offsets), _p(num_append),
                                    _p(k_pool), _p(v_pool), _p(page_table), _p(cached_lens), _p(free_pages),
                                    _p(free_count), _p(workspace), workspace.numel(), _stream(stream))
    _lib.check(rc, "hstu_kv_append")
    return workspace


def hstu_kv_evict(evict_mask, k_pool, page_table, cached_lens, free_pages, free_count, *, workspace=None,
                  stream=None):
    """Returns the pages of every user with evict_mask[u] != 0 to the free stack; in place."""
    _kv_check(k_pool, page_table, cached_lens, free_pages, free_count)
    _need_cuda("evict_mask", evict_mask, torch.int32)
    p = kv_params(k_pool, page_table)
    if workspace is None:
        workspace = torch.empty(hstu_kv_workspace_size(p), dtype=torch.uint8, device=k_pool.device)
    rc = _lib.load().hstu_kv_evict(ctypes.byref(p), _p(evict_mask), _p(page_table), _p(cached_lens),
                                   _p(free_pages), _p(free_count), _p(workspace), workspace.numel(),
                                   _stream(stream))
    _lib.check(rc, "hstu_kv_evict")
    return workspace


def hstu_mfalcon_workspace_size(p: _lib.AttnParams, microbatch: int, num_splits: int, hist_tokens: int) -> int:
    return int(_lib.load().hstu_mfalcon_workspace_size(ctypes.byref(p), microbatch, num_splits, hist_tokens))


def hstu_mfalcon_fwd(q_c, k_c, v_c, u_c, cand_offsets, hist_timestamps, hist_ts_offsets, cand_timestamps,
                     rab_pos, rab_ts, k_pool, v_pool, kv_page_table, cached_lens, *, n_max: int, microbatch: int,
                     max_candidates: int, max_cached_len: Optional[int] = None, alpha: Optional[float] = None,
                     ln_gamma=None, ln_beta=None, ln_eps: float = 1e-5, num_splits: Optional[int] = None,
                     out=None, workspace=None, force_simt: bool = False, precise_silu: bool = False,
                     stream=None):
    """M-FALCON: every candidate attends to its user's cached history and itself;
    candidates go through the paged forward `microbatch` per user at a time."""
    T, H, d = q_c.shape
    dt = q_c.dtype
    for name, t in (("q_c", q_c), ("k_c", k_c), ("v_c", v_c), ("u_c", u_c), ("k_pool", k_pool), ("v_pool", v_pool)):
        _need_cuda(name, t, dt)
    for name, t in (("cand_offsets", cand_offsets), ("hist_ts_offsets", hist_ts_offsets),
                    ("kv_page_table", kv_page_table), ("cached_lens", cached_lens)):
        _need_cuda(name, t, torch.int32)
    _need_cuda("hist_timestamps", hist_timestamps, torch.int64)
    _need_cuda("cand_timestamps", cand_timestamps, torch.int64)
    qs = _rows_view("q_c", q_c, H, d)
    if _rows_view("k_c", k_c, H, d) != qs or _rows_view("v_c", v_c, H, d) != qs:
        raise ValueError("q_c, k_c and v_c must share one token stride")
    us = _rows_view("u_c", u_c, H, d)
    B = cand_offsets.numel() - 1
    num_pages, _, page_size, _ = k_pool.shape
    mc = n_max if max_cached_len is None else max_cached_len
    flags = (_lib.F_FORCE_SIMT if force_simt else 0) | (_lib.F_PRECISE_SILU if precise_silu else 0)
    params = attn_params(batch=B, num_heads=H, head_dim=d, n_max=n_max, total_tokens=T,
                         max_seq_len=min(n_max, mc + microbatch), dtype=dt, alpha=alpha,
                         num_ts_buckets=rab_ts.numel(), qkv_stride=qs, u_stride=us, ln_eps=ln_eps, flags=flags)
    if num_splits is None:
        num_splits = hstu_attn_paged_default_splits(
            attn_params(batch=B, num_heads=H, head_dim=d, n_max=n_max, total_tokens=B * microbatch,
                        max_seq_len=n_max, dtype=dt), mc)
    if out is None:
        out = torch.empty(T, H * d, dtype=dt, device=q_c.device)
    hist_tokens = hist_timestamps.numel()
    if workspace is None:
        workspace = torch.empty(hstu_mfalcon_workspace_size(params, microbatch, num_splits, hist_tokens),
                                dtype=torch.uint8, device=q_c.device)
    rc = _lib.load().hstu_mfalcon_fwd(
        ctypes.byref(params), _p(q_c), _p(k_c), _p(v_c), _p(u_c), _p(cand_offsets), _p(hist_timestamps),
        _p(hist_ts_offsets), hist_tokens, _p(cand_timestamps), _p(rab_pos), _p(rab_ts), _p(ln_gamma), _p(ln_beta),
        _p(k_pool), _p(v_pool), num_pages, _p(kv_page_table), kv_page_table.shape[1], page_size, _p(cached_lens),
        max_candidates, microbatch, num_splits, _p(out), _p(workspace), workspace.numel(), _stream(stream))
    _lib.check(rc, "hstu_mfalcon_fwd")
    return out, workspace


def hstu_attn_bwd(q, k, v, seq_offsets, timestamps, rab_pos, rab_ts, d_o, *, n_max: int,
                  alpha: Optional[float] = None, num_candidates=None, max_seq_len: Optional[int] = None,
                  workspace=None, stream=None, force_simt: bool = False):
    """Gradients of the raw per-head output o = A V: returns d_q, d_k, d_v [T, H, d]
    and d_rab_pos, d_rab_ts (all fp32).  bf16 inputs with d = 128 run on the
    tensor cores (bf16 GEMM operands); force_simt keeps them on the fp32
    CUDA-core kernel."""
    T, H, d = q.shape
    dt = q.dtype
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need_cuda(name, t, dt)
    _need_cuda("d_o", d_o, torch.float32)
    _need_cuda("seq_offsets", seq_offsets, torch.int32)
    _need_cuda("timestamps", timestamps, torch.int64)
    _need_cuda("num_candidates", num_candidates, torch.int32)
    _need_cuda("rab_pos", rab_pos, torch.float32)
    _need_cuda("rab_ts", rab_ts, torch.float32)
    if not d_o.is_contiguous() or d_o.shape != q.shape:
        raise ValueError("d_o must be a contiguous [T, H, d] tensor")
    qs = _rows_view("q", q, H, d)
    if _rows_view("k", k, H, d) != qs or _rows_view("v", v, H, d) != qs:
        raise ValueError("q, k and v must share one token stride")
    params = attn_params(batch=seq_offsets.numel() - 1, num_heads=H, head_dim=d, n_max=n_max, total_tokens=T,
                         max_seq_len=n_max if max_seq_len is None else max_seq_len, dtype=dt, alpha=alpha,
                         num_ts_buckets=rab_ts.numel(), qkv_stride=qs,
                         flags=_lib.F_FORCE_SIMT if force_simt else 0)
    grads = [torch.empty(T, H, d, dtype=torch.float32, device=q.device) for _ in range(3)]
    d_rp = torch.empty_like(rab_pos)
    d_rt = torch.empty_like(rab_ts)
    if workspace is None:
        workspace = torch.empty(int(_lib.load().hstu_attn_bwd_workspace_size(ctypes.byref(params))),
                                dtype=torch.uint8, device=q.device)
    rc = _lib.load().hstu_attn_bwd(ctypes.byref(params), _p(q), _p(k), _p(v), _p(seq_offsets), _p(timestamps),
                                   _p(num_candidates), _p(rab_pos), _p(rab_ts), _p(d_o), _p(grads[0]),
                                   _p(grads[1]), _p(grads[2]), _p(d_rp), _p(d_rt), _p(workspace),
                                   workspace.numel(), _stream(stream))
    _lib.check(rc, "hstu_attn_bwd")
    return grads[0], grads[1], grads[2], d_rp, d_rt, workspace
