"""CPU-only checks of the C ABI: the library builds, loads, exports every
symbol include/hstu.h declares, and rejects bad host arguments before it
touches a GPU."""
import ctypes
import os
import re
import subprocess

import pytest

import generative_recommender_attention_jagged_b200 as hstu
from generative_recommender_attention_jagged_b200 import _lib, build as hbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hstu.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\**\s*(hstu_[a-z_0-9]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    hbuild.build()
    return _lib.load()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("hstu_attn_fwd", "hstu_attn_fwd_paged", "hstu_ts_bucket", "hstu_attn_workspace_size",
                     "hstu_check_device_error", "hstu_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(lib, n)


def test_params_struct_matches_header(lib):
    assert ctypes.sizeof(_lib.AttnParams) == 13 * 4


def test_status_strings(lib):
    assert hstu.hstu_status_string(0) == "HSTU_OK"
    for code in range(-10, 0):
        assert hstu.hstu_status_string(code).startswith(_lib.STATUS_NAMES[code])
    assert hstu.hstu_version() == 100


def params(**kw):
    base = dict(batch=2, num_heads=4, head_dim=128, n_max=1024, total_tokens=300, max_seq_len=200,
                dtype=__import__("torch").bfloat16)
    base.update(kw)
    return hstu.attn_params(**base)


def test_workspace_size_grows_with_tokens_and_splits(lib):
    small = hstu.hstu_attn_workspace_size(params())
    big = hstu.hstu_attn_workspace_size(params(total_tokens=3000))
    assert 0 < small < big
    assert small >= 256 + 300 * 512 * 4
    assert hstu.hstu_attn_paged_workspace_size(params(), 4) >= hstu.hstu_attn_paged_workspace_size(params(), 1)


@pytest.mark.parametrize("bad", [dict(batch=0), dict(num_heads=0), dict(n_max=0), dict(num_ts_buckets=129),
                                 dict(head_dim=300), dict(flags=0x1000)])
def test_bad_params_rejected_on_host(lib, bad):
    p = params(**bad)
    assert lib.hstu_attn_workspace_size(ctypes.byref(p)) == 0
    rc = lib.hstu_attn_fwd(ctypes.byref(p), *([None] * 13), 0, None)
    assert rc in (-1, -2)


def test_null_pointers_rejected_on_host(lib):
    p = params()
    rc = lib.hstu_attn_fwd(ctypes.byref(p), *([None] * 13), 0, None)
    assert rc == -1
    rc = lib.hstu_attn_fwd_paged(ctypes.byref(p), *([None] * 14), 1, None, 1, 32, None, 1, None, None, 0, None)
    assert rc == -1


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="hands fake device pointers to the library; run only where no GPU can see them")
def test_empty_batch_accepts_null_token_arrays_on_host(lib):
    """With T = 0 the token-indexed arrays may be NULL: the host checks pass
    and the call gets as far as its first CUDA call (which fails here, with no
    GPU); with T > 0 the same NULLs are an invalid argument."""
    fake = ctypes.c_void_p(0x1000)
    for total, want_invalid in ((0, False), (5, True)):
        p = params(total_tokens=total)
        args = [None] * 13
        args[4], args[7], args[8], args[12] = fake, fake, fake, fake  # offsets, rab_pos, rab_ts, workspace
        rc = lib.hstu_attn_fwd(ctypes.byref(p), *args, 1 << 30, None)
        assert (rc == -1) == want_invalid, (total, rc)
        bargs = [None] * 15
        for i in (3, 6, 7, 12, 13, 14):  # offsets, rab_pos, rab_ts, d_rab_pos, d_rab_ts, workspace
            bargs[i] = fake
        rc = lib.hstu_attn_bwd(ctypes.byref(p), *bargs, 1 << 30, None)
        assert (rc == -1) == want_invalid, (total, rc)


def test_misaligned_pointer_rejected_on_host(lib):
    p = params()
    fake = [ctypes.c_void_p(0x1000)] * 13
    fake[0] = ctypes.c_void_p(0x1008)  # q not 16-byte aligned
    rc = lib.hstu_attn_fwd(ctypes.byref(p), *fake, 1 << 30, None)
    assert rc == -3


def test_small_workspace_rejected_on_host(lib):
    p = params(flags=_lib.F_FORCE_SIMT)
    fake = [ctypes.c_void_p(0x1000)] * 13
    rc = lib.hstu_attn_fwd(ctypes.byref(p), *fake, 64, None)
    assert rc == -5


def test_bucket_kernel_rejects_bad_args_on_host(lib):
    assert lib.hstu_ts_bucket(None, -1, 128, None, None) == -1
    assert lib.hstu_ts_bucket(None, 10, 128, None, None) == -1
    assert lib.hstu_ts_bucket(None, 0, 0, None, None) == -1


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(4, 1, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        hstu.hstu_attn_fwd(q, q, q, q.view(4, 128), torch.tensor([0, 4], dtype=torch.int32),
                           torch.zeros(4, dtype=torch.int64), torch.zeros(7), torch.zeros(128), n_max=4)


# ---- linear glue (f1 / f2) --------------------------------------------------
def test_linear_params_struct_matches_header(lib):
    # int64 rows, int32 d_in, int32 d_out, int64 x_stride, int64 out_stride, int32 dtype, uint32 flags
    assert ctypes.sizeof(_lib.LinearParams) == 40


def lin(**kw):
    base = dict(rows=300, d_in=512, d_out=2048, x_stride=0, out_stride=0, dtype=_lib.DT_BF16, flags=0)
    base.update(kw)
    return _lib.LinearParams(**base)


@pytest.mark.parametrize("name", ["hstu_linear", "hstu_layer_f1", "hstu_layer_f2"])
def test_linear_rejects_bad_args_on_host(lib, name):
    fn = getattr(lib, name)
    a = ctypes.c_void_p(0x1000)
    ws = 1 << 26
    assert fn(None, a, a, None, a, a, ws, None) == -1
    assert fn(ctypes.byref(lin(rows=-1)), a, a, None, a, a, ws, None) == -1
    assert fn(ctypes.byref(lin(d_in=0)), a, a, None, a, a, ws, None) == -1
    assert fn(ctypes.byref(lin(dtype=7)), a, a, None, a, a, ws, None) == -1
    assert fn(ctypes.byref(lin(flags=0x8)), a, a, None, a, a, ws, None) == -1
    assert fn(ctypes.byref(lin(x_stride=100)), a, a, None, a, a, ws, None) == -1   # stride < d_in
    assert fn(ctypes.byref(lin()), None, a, None, a, a, ws, None) == -1
    assert fn(ctypes.byref(lin(d_out=2044)), a, a, None, a, a, ws, None) == -3
    assert fn(ctypes.byref(lin()), ctypes.c_void_p(0x1008), a, None, a, a, ws, None) == -3
    assert fn(ctypes.byref(lin()), a, a, None, a, a, 1024, None) == -5
    # no rows: nothing to do, no pointer is looked at
    assert fn(ctypes.byref(lin(rows=0)), None, None, None, None, None, 0, None) == 0


def test_linear_workspace_size(lib):
    assert hstu.hstu_linear_workspace_size() >= 1 << 20


# ---- KV cache write side ----------------------------------------------------
def test_kv_params_struct_matches_header(lib):
    assert ctypes.sizeof(_lib.KvParams) == 9 * 4


def kvp(**kw):
    base = dict(batch=3, num_heads=4, head_dim=128, page_size=32, num_pages=100, max_pages_per_user=8,
                kv_stride=0, total_new=50, dtype=_lib.DT_BF16)
    base.update(kw)
    return _lib.KvParams(**base)


def test_kv_rejects_bad_args_on_host(lib):
    a = ctypes.c_void_p(0x1000)
    ws = 1 << 20
    assert lib.hstu_kv_workspace_size(ctypes.byref(kvp())) >= 256 + 3 * 8
    assert lib.hstu_kv_workspace_size(ctypes.byref(kvp(batch=0))) == 0
    assert lib.hstu_kv_append(None, *([a] * 11), ws, None) == -1
    assert lib.hstu_kv_append(ctypes.byref(kvp(page_size=0)), *([a] * 11), ws, None) == -1
    assert lib.hstu_kv_append(ctypes.byref(kvp(dtype=5)), *([a] * 11), ws, None) == -1
    assert lib.hstu_kv_append(ctypes.byref(kvp()), None, *([a] * 10), ws, None) == -1
    assert lib.hstu_kv_append(ctypes.byref(kvp(kv_stride=100)), *([a] * 11), ws, None) == -1  # < H*d
    assert lib.hstu_kv_append(ctypes.byref(kvp(head_dim=4)), *([a] * 11), ws, None) == -3      # 8-byte rows
    assert lib.hstu_kv_append(ctypes.byref(kvp()), ctypes.c_void_p(0x1004), *([a] * 10), ws, None) == -3
    assert lib.hstu_kv_append(ctypes.byref(kvp()), *([a] * 11), 16, None) == -5
    assert lib.hstu_kv_evict(ctypes.byref(kvp()), None, a, a, a, a, a, ws, None) == -1
    assert lib.hstu_kv_evict(ctypes.byref(kvp()), *([a] * 6), 16, None) == -5


def test_mfalcon_rejects_bad_args_on_host(lib):
    p = params()
    a = ctypes.c_void_p(0x1000)
    ws = 1 << 30
    full = [a] * 7
    assert lib.hstu_mfalcon_workspace_size(ctypes.byref(p), 0, 1, 100) == 0
    assert lib.hstu_mfalcon_workspace_size(ctypes.byref(p), 128, 1, 100) > 0
    args = lambda mb=128, q=a: ([ctypes.byref(p), q] + full[1:] + [100, a] + [a] * 6 +
                                [10, a, 4, 32, a, 256, mb, 1, a, a, ws, None])
    assert lib.hstu_mfalcon_fwd(*args(mb=0)) == -1
    assert lib.hstu_mfalcon_fwd(*args(q=None)) == -1
    assert lib.hstu_mfalcon_fwd(*args(q=ctypes.c_void_p(0x1008))) == -3


@pytest.mark.parametrize("bad,code", [(dict(batch=0), -1), (dict(num_ts_buckets=129), -2), (dict(head_dim=300), -2),
                                      (dict(dtype=__import__("torch").bfloat16, num_heads=4, head_dim=3), -3)])
def test_static_ws_entry_returns_the_workspace_entry_codes(lib, bad, code):
    # the allocation-free entry point checks the parameters exactly as
    # hstu_attn_fwd does (no GPU is touched: the checks fail first)
    p = params(**bad)
    rc_ws = lib.hstu_attn_fwd(ctypes.byref(p), *([None] * 13), 0, None)
    rc_static = lib.hstu_attn_fwd_static_ws(ctypes.byref(p), *([None] * 13))
    assert rc_ws == code and rc_static == code
