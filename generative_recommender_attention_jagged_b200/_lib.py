"""ctypes view of libhstu.so (the C ABI in include/hstu.h).

Argument marshalling only: every step of the computation runs in the CUDA
library.  Loading fails loudly when the library is missing; there is no
fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhstu.so")

HSTU_OK = 0
STATUS_NAMES = {
    0: "HSTU_OK", -1: "HSTU_ERR_INVALID_ARG", -2: "HSTU_ERR_UNSUPPORTED", -3: "HSTU_ERR_ALIGNMENT",
    -4: "HSTU_ERR_LENGTH", -5: "HSTU_ERR_WORKSPACE", -6: "HSTU_ERR_CUDA", -7: "HSTU_ERR_TIMEOUT",
    -8: "HSTU_ERR_UNSORTED", -9: "HSTU_ERR_PAGE", -10: "HSTU_ERR_POOL",
}

DT_F32 = 0
DT_BF16 = 1

F_FORCE_SIMT = 0x1
F_OUTPUT_RAW_AV = 0x2
F_PRECISE_SILU = 0x4
F_STAGE_PLAN = 0x10
F_STAGE_ATTN = 0x20
F_STAGE_EPILOGUE = 0x40

LIN_SILU = 0x1
LIN_CUBLAS = 0x2


class AttnParams(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("num_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("n_max", ctypes.c_int32),
        ("num_ts_buckets", ctypes.c_int32),
        ("total_tokens", ctypes.c_int32),
        ("max_seq_len", ctypes.c_int32),
        ("qkv_stride", ctypes.c_int32),
        ("u_stride", ctypes.c_int32),
        ("alpha", ctypes.c_float),
        ("ln_eps", ctypes.c_float),
        ("dtype", ctypes.c_int32),
        ("flags", ctypes.c_uint32),
    ]


class LinearParams(ctypes.Structure):
    _fields_ = [
        ("rows", ctypes.c_int64),
        ("d_in", ctypes.c_int32),
        ("d_out", ctypes.c_int32),
        ("x_stride", ctypes.c_int64),
        ("out_stride", ctypes.c_int64),
        ("dtype", ctypes.c_int32),
        ("flags", ctypes.c_uint32),
    ]


class KvParams(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("num_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("max_pages_per_user", ctypes.c_int32),
        ("kv_stride", ctypes.c_int32),
        ("total_new", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
    ]


class HstuError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libhstu.so is not built ({LIB_PATH}); run __graft_entry__.build()")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    PP = ctypes.POINTER(AttnParams)
    i32, i64, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    lib.hstu_attn_workspace_size.argtypes = [PP]
    lib.hstu_attn_workspace_size.restype = sz
    lib.hstu_attn_fwd.argtypes = [PP] + [P] * 13 + [sz, P]
    lib.hstu_attn_fwd.restype = ctypes.c_int
    lib.hstu_attn_paged_workspace_size.argtypes = [PP, i32]
    lib.hstu_attn_paged_workspace_size.restype = sz
    lib.hstu_attn_paged_default_splits.argtypes = [PP, i32]
    lib.hstu_attn_paged_default_splits.restype = i32
    lib.hstu_attn_fwd_paged.argtypes = ([PP] + [P] * 14 + [i32, P, i32, i32, P, i32, P, P, sz, P])
    lib.hstu_attn_fwd_paged.restype = ctypes.c_int
    lib.hstu_ts_bucket.argtypes = [P, i64, i32, P, P]
    lib.hstu_ts_bucket.restype = ctypes.c_int
    lib.hstu_check_device_error.argtypes = [P, P]
    lib.hstu_check_device_error.restype = ctypes.c_int
    lib.hstu_status_string.argtypes = [ctypes.c_int]
    lib.hstu_status_string.restype = ctypes.c_char_p
    LP = ctypes.POINTER(LinearParams)
    lib.hstu_linear_workspace_size.argtypes = [LP]
    lib.hstu_linear_workspace_size.restype = sz
    for name in ("hstu_linear", "hstu_layer_f1", "hstu_layer_f2"):
        fn = getattr(lib, name)
        fn.argtypes = [LP, P, P, P, P, P, sz, P]
        fn.restype = ctypes.c_int
    lib.hstu_attn_fwd_static_ws.argtypes = [PP] + [P] * 13
    lib.hstu_attn_fwd_static_ws.restype = ctypes.c_int
    lib.hstu_static_ws_check_device_error.argtypes = [P]
    lib.hstu_static_ws_check_device_error.restype = ctypes.c_int
    lib.hstu_attn_bwd_workspace_size.argtypes = [PP]
    lib.hstu_attn_bwd_workspace_size.restype = sz
    lib.hstu_attn_bwd.argtypes = [PP] + [P] * 15 + [sz, P]
    lib.hstu_attn_bwd.restype = ctypes.c_int
    lib.hstu_mfalcon_workspace_size.argtypes = [PP, i32, i32, i64]
    lib.hstu_mfalcon_workspace_size.restype = sz
    lib.hstu_mfalcon_fwd.argtypes = ([PP] + [P] * 7 + [i64, P] + [P] * 6 + [i32, P, i32, i32, P, i32, i32, i32, P, P,
                                                                         sz, P])
    lib.hstu_mfalcon_fwd.restype = ctypes.c_int
    KP = ctypes.POINTER(KvParams)
    lib.hstu_kv_workspace_size.argtypes = [KP]
    lib.hstu_kv_workspace_size.restype = sz
    lib.hstu_kv_append.argtypes = [KP] + [P] * 11 + [sz, P]
    lib.hstu_kv_append.restype = ctypes.c_int
    lib.hstu_kv_evict.argtypes = [KP] + [P] * 6 + [sz, P]
    lib.hstu_kv_evict.restype = ctypes.c_int
    lib.hstu_version.argtypes = []
    lib.hstu_version.restype = ctypes.c_int
    _lib = lib
    return lib


def check(status: int, where: str) -> None:
    if status != HSTU_OK:
        raise HstuError(status, where)
