"""The C ABI boundary on the CPU: libear loads, exports every symbol that
include/ear.h declares, and its host-side validation rejects bad arguments
before any CUDA call (so these run without a GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

from clustered_block_sparse_b200 import _native as N
from clustered_block_sparse_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return N.lib()


def declared_symbols():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            names |= set(re.findall(r"EAR_API\s+[\w\s\*]+?\b(ear_\w+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert {"ear_kmeans", "ear_permute", "ear_probe", "ear_route", "ear_attention"} <= names
    out = subprocess.run(["nm", "-D", "--defined-only", N.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (ear_\w+)", out))
    assert names <= exported, names - exported
    for n in names:
        assert hasattr(lib, n)


def test_library_needs_no_shared_cuda_runtime():
    out = subprocess.run(["ldd", N.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcudart" not in out


def test_status_strings(lib):
    for code in range(7):
        assert lib.ear_status_string(code).decode().startswith("EAR_")


def test_workspace_sizes_grow_with_problem(lib):
    small = N.workspace_bytes(N.EAR_OP_KMEANS, 1, 1024, 0, 64, 16, 0)
    big = N.workspace_bytes(N.EAR_OP_KMEANS, 40, 75600, 0, 128, 500, 0)
    assert 0 < small < big
    assert N.workspace_bytes(N.EAR_OP_ATTENTION, 2, 1000, 1000, 128, 10, 20) > 0
    out = ctypes.c_size_t(0)
    assert lib.ear_workspace_bytes(0, -1, 1, 1, 64, 1, 1, ctypes.byref(out)) == N.EAR_ERR_ARG
    assert lib.ear_workspace_bytes(0, 1, 1, 1, 64, 1, 1, None) == N.EAR_ERR_ARG


FAKE = ctypes.c_void_p(0x10000)        # aligned, never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p(0x10004)


def kmeans(lib, X=FAKE, dtype=N.EAR_BF16, bh=1, n=1024, d=128, c=16, iters=1, ws=None, nb=0):
    return lib.ear_kmeans(X, dtype, bh, n, d, c, iters, FAKE, FAKE, FAKE, FAKE, ws, nb, None)


def test_kmeans_validation(lib):
    assert kmeans(lib, X=None) == N.EAR_ERR_ARG
    assert kmeans(lib, X=MISALIGNED) == N.EAR_ERR_ARG
    assert kmeans(lib, dtype=7) == N.EAR_ERR_ARG
    assert kmeans(lib, c=0) == N.EAR_ERR_ARG
    assert kmeans(lib, c=2000, n=1024) == N.EAR_ERR_ARG      # more clusters than rows
    assert kmeans(lib, iters=0) == N.EAR_ERR_ARG
    assert kmeans(lib, d=96) == N.EAR_ERR_UNSUPPORTED
    assert kmeans(lib, bh=70000) == N.EAR_ERR_UNSUPPORTED
    assert kmeans(lib, ws=FAKE, nb=16) == N.EAR_ERR_WORKSPACE


def test_permute_validation(lib):
    f = lib.ear_permute
    assert f(None, 1, 100, 4, FAKE, FAKE, None, None, 0, 0, None, FAKE, 1 << 30, None) == N.EAR_ERR_ARG
    # X_perm without X
    assert f(FAKE, 1, 100, 4, FAKE, FAKE, None, FAKE, 0, 0, None, FAKE, 1 << 30, None) == N.EAR_ERR_ARG
    assert f(FAKE, 1, 100, 4, FAKE, FAKE, FAKE, FAKE, 1, 80, None, FAKE, 1 << 30, None) == N.EAR_ERR_UNSUPPORTED
    assert f(FAKE, 1, 100, 4, FAKE, FAKE, None, None, 0, 0, None, FAKE, 4, None) == N.EAR_ERR_WORKSPACE


def test_permute_apply_validation(lib):
    f = lib.ear_permute_apply
    assert f(None, FAKE, 1, 100, 4, FAKE, FAKE, 1, 128, None, None) == N.EAR_ERR_ARG
    assert f(FAKE, FAKE, 1, 100, 4, None, FAKE, 1, 128, None, None) == N.EAR_ERR_ARG
    assert f(FAKE, FAKE, 1, 100, 4, FAKE, FAKE, 1, 128, MISALIGNED, None) == N.EAR_ERR_ARG
    assert f(FAKE, FAKE, 1, 100, 4, FAKE, FAKE, 1, 96, None, None) == N.EAR_ERR_UNSUPPORTED
    # X_perm may be left out only when the means are asked for
    assert f(FAKE, FAKE, 1, 100, 4, FAKE, None, 1, 128, None, None) == N.EAR_ERR_ARG
    assert f(FAKE, FAKE, 1, 100, 4, FAKE, None, 1, 96, FAKE, None) == N.EAR_ERR_UNSUPPORTED


def test_probe_gather_validation(lib):
    f = lib.ear_probe_gather

    def call(K=FAKE, kp=FAKE, d=128, mode=0, V=None, vc=None):
        return f(FAKE, FAKE, FAKE, K, kp, 1, FAKE, 1, 100, d, 4, 4, ctypes.c_float(0.1), mode, V,
                 vc, FAKE, None, 0, None)
    assert call(kp=None) == N.EAR_ERR_ARG
    assert call(kp=MISALIGNED) == N.EAR_ERR_ARG
    assert call(K=None) == N.EAR_ERR_ARG
    assert call(mode=3) == N.EAR_ERR_ARG
    assert call(mode=N.EAR_PROBE_VALUE) == N.EAR_ERR_ARG          # values missing
    assert call(d=32) == N.EAR_ERR_UNSUPPORTED
    assert call(mode=N.EAR_PROBE_VALUE, V=FAKE, vc=FAKE, d=32) == N.EAR_ERR_UNSUPPORTED


def test_probe_validation(lib):
    f = lib.ear_probe

    def call(K=FAKE, dtype=1, d=128, scale=0.1, mode=0, V=None, vc=None):
        return f(FAKE, FAKE, FAKE, K, dtype, FAKE, 1, 100, d, 4, 4, ctypes.c_float(scale), mode, V,
                 vc, FAKE, None, 0, None)
    assert call(scale=float("nan")) == N.EAR_ERR_ARG
    assert call(K=None) == N.EAR_ERR_ARG
    assert call(d=32) == N.EAR_ERR_UNSUPPORTED
    assert call(mode=3) == N.EAR_ERR_ARG
    assert call(mode=N.EAR_PROBE_VALUE) == N.EAR_ERR_ARG          # values missing
    assert call(mode=N.EAR_PROBE_WEIGHTS, dtype=0) == N.EAR_ERR_UNSUPPORTED  # fp32 keys


def test_route_validation(lib):
    f = lib.ear_route
    args = lambda dens, mode: (FAKE, FAKE, FAKE, 1, 100, 100, 4, 4, ctypes.c_double(dens), mode,
                               FAKE, FAKE, FAKE, FAKE, None, 0, None)
    assert f(*args(-0.1, 0)) == N.EAR_ERR_ARG
    assert f(*args(1.5, 0)) == N.EAR_ERR_ARG
    assert f(*args(float("nan"), 0)) == N.EAR_ERR_ARG
    assert f(*args(0.5, 2)) == N.EAR_ERR_ARG


def test_attention_validation(lib):
    f = lib.ear_attention

    def call(flags=1, d=128, lse=None, scale=0.1):
        return f(FAKE, FAKE, FAKE, 1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 100, 100,
                 d, 4, 4, ctypes.c_float(scale), flags, FAKE, lse, FAKE, 1 << 30, None)
    assert call(flags=4) == N.EAR_ERR_ARG
    assert call(lse=MISALIGNED) == N.EAR_ERR_ARG
    assert call(scale=float("inf")) == N.EAR_ERR_ARG
    assert call(d=256) == N.EAR_ERR_UNSUPPORTED


def test_attention_gather_validation(lib):
    f = lib.ear_attention_gather

    def call(kp=FAKE, flags=1, d=128, Q=FAKE):
        return f(Q, FAKE, FAKE, 1, FAKE, FAKE, FAKE, kp, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 100, 100,
                 d, 4, 4, ctypes.c_float(0.1), flags, FAKE, None, FAKE, 1 << 30, None)
    assert call(kp=None) == N.EAR_ERR_ARG
    assert call(kp=MISALIGNED) == N.EAR_ERR_ARG
    assert call(Q=None) == N.EAR_ERR_ARG
    assert call(flags=4) == N.EAR_ERR_ARG
    assert call(d=256) == N.EAR_ERR_UNSUPPORTED


def test_status_query_rejects_null(lib):
    assert lib.ear_get_device_status(None, None) == N.EAR_ERR_ARG


def test_route_rows_and_budget_validation(lib):
    f = lib.ear_route_rows
    assert f(FAKE, FAKE, FAKE, 1, 4, 9000, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20,
             None) == N.EAR_ERR_UNSUPPORTED                       # C_k above 8192
    assert f(None, FAKE, FAKE, 1, 4, 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20,
             None) == N.EAR_ERR_ARG
    assert f(FAKE, FAKE, FAKE, 1, 4, 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 8,
             None) == N.EAR_ERR_WORKSPACE
    g = lib.ear_topp_budget
    assert g(FAKE, FAKE, FAKE, FAKE, 1, 128, 4, 4, ctypes.c_float(0.1), ctypes.c_double(1.5),
             FAKE, None) == N.EAR_ERR_ARG
    assert g(FAKE, FAKE, FAKE, FAKE, 1, 96, 4, 4, ctypes.c_float(0.1), ctypes.c_double(0.5),
             FAKE, None) == N.EAR_ERR_UNSUPPORTED
    u = lib.ear_uniform_budget
    assert u(FAKE, 1, 4, 100, ctypes.c_double(-0.5), FAKE, None) == N.EAR_ERR_ARG
    assert u(None, 1, 4, 100, ctypes.c_double(0.5), FAKE, None) == N.EAR_ERR_ARG
