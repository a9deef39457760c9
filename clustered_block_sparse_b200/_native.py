"""ctypes handle on libear.so (the C ABI in include/ear.h).

The library must have been built in-tree (``python -m
clustered_block_sparse_b200.build``); there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libear.so")

EAR_OK, EAR_ERR_ARG, EAR_ERR_UNSUPPORTED, EAR_ERR_WORKSPACE, EAR_ERR_CUDA, EAR_ERR_TIMEOUT, \
    EAR_ERR_DEVICE = range(7)
EAR_F32, EAR_BF16 = 0, 1
EAR_OP_KMEANS, EAR_OP_PERMUTE, EAR_OP_PROBE, EAR_OP_ROUTE, EAR_OP_ATTENTION, \
    EAR_OP_ROUTE_ROWS = range(6)
EAR_COMPENSATE = 1
EAR_PROBE_LOGIT, EAR_PROBE_WEIGHTS, EAR_PROBE_VALUE = 0, 1, 2

EXPORTED = ("ear_status_string", "ear_workspace_bytes", "ear_kmeans", "ear_permute",
            "ear_permute_apply", "ear_permute_static", "ear_probe", "ear_probe_gather", "ear_route",
            "ear_attention", "ear_attention_gather",
            "ear_route_rows", "ear_topp_budget", "ear_uniform_budget", "ear_cluster_stats",
            "ear_normalizer_change",
            "ear_get_device_status", "ear_launch_count")
PERMUTE_STATIC_MAX_BYTES = 8 << 20

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_lib = None


class EarError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = lib().ear_status_string(status).decode() if _lib is not None else str(status)
        super().__init__(f"{fn} failed: {msg}")


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"libear.so is not built ({LIB_PATH}); run `python -m clustered_block_sparse_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    L.ear_status_string.argtypes = [ctypes.c_int]
    L.ear_status_string.restype = ctypes.c_char_p
    L.ear_workspace_bytes.argtypes = [ctypes.c_int, _i64, _i64, _i64, _i32, _i32, _i32,
                                      ctypes.POINTER(ctypes.c_size_t)]
    L.ear_kmeans.argtypes = [_vp, ctypes.c_int, _i64, _i64, _i32, _i32, _i32, _vp, _vp, _vp, _vp,
                             _vp, ctypes.c_size_t, _vp]
    L.ear_permute.argtypes = [_vp, _i64, _i64, _i32, _vp, _vp, _vp, _vp, ctypes.c_int, _i32, _vp,
                              _vp, ctypes.c_size_t, _vp]
    L.ear_permute_apply.argtypes = [_vp, _vp, _i64, _i64, _i32, _vp, _vp, ctypes.c_int, _i32, _vp,
                                    _vp]
    L.ear_permute_static.argtypes = [_vp, _i64, _i64, _i32, _vp, _vp, _vp, _vp, ctypes.c_int,
                                     _i32, _vp, _vp]
    L.ear_probe.argtypes = [_vp, _vp, _vp, _vp, ctypes.c_int, _vp, _i64, _i64, _i32, _i32, _i32,
                            ctypes.c_float, _i32, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
    L.ear_probe_gather.argtypes = [_vp, _vp, _vp, _vp, _vp, ctypes.c_int, _vp, _i64, _i64, _i32,
                                   _i32, _i32, ctypes.c_float, _i32, _vp, _vp, _vp, _vp,
                                   ctypes.c_size_t, _vp]
    L.ear_route.argtypes = [_vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, ctypes.c_double, _i32,
                            _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
    L.ear_route_rows.argtypes = [_vp, _vp, _vp, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp,
                                 ctypes.c_size_t, _vp]
    L.ear_topp_budget.argtypes = [_vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, ctypes.c_float,
                                  ctypes.c_double, _vp, _vp]
    L.ear_uniform_budget.argtypes = [_vp, _i64, _i32, _i64, ctypes.c_double, _vp, _vp]
    L.ear_cluster_stats.argtypes = [_vp, ctypes.c_int, _vp, _vp, _i64, _i64, _i32, _i32, _vp, _vp,
                                    _vp]
    L.ear_normalizer_change.argtypes = [_vp, _vp, _i64, _i64, _vp, _vp]
    L.ear_attention.argtypes = [_vp, _vp, _vp, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                _vp, _i64, _i64, _i64, _i32, _i32, _i32, ctypes.c_float, _i32,
                                _vp, _vp, _vp, ctypes.c_size_t, _vp]
    L.ear_attention_gather.argtypes = [_vp, _vp, _vp, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp,
                                       _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32,
                                       ctypes.c_float, _i32, _vp, _vp, _vp, ctypes.c_size_t, _vp]
    L.ear_get_device_status.argtypes = [ctypes.POINTER(ctypes.c_int32), _vp]
    L.ear_launch_count.argtypes = []
    L.ear_launch_count.restype = ctypes.c_uint64
    for name in ("ear_workspace_bytes", "ear_kmeans", "ear_permute", "ear_permute_apply",
                 "ear_permute_static",
                 "ear_probe", "ear_probe_gather", "ear_route", "ear_route_rows", "ear_topp_budget",
                 "ear_uniform_budget", "ear_cluster_stats", "ear_normalizer_change",
                 "ear_attention", "ear_attention_gather", "ear_get_device_status"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def check(fn: str, status: int) -> None:
    if status != EAR_OK:
        raise EarError(fn, status)


def workspace_bytes(op: int, bh: int, n_q: int, n_k: int, d: int, c_q: int, c_k: int) -> int:
    out = ctypes.c_size_t(0)
    check("ear_workspace_bytes", lib().ear_workspace_bytes(op, bh, n_q, n_k, d, c_q, c_k,
                                                           ctypes.byref(out)))
    return int(out.value)


def launch_count() -> int:
    return int(lib().ear_launch_count())
