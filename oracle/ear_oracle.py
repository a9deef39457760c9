"""ctypes front-end of the fp64 C++ oracle (test infrastructure only).

Each function takes numpy arrays for ONE (batch, head) slice in original token
order, upcasts them to float64 and calls the C++ routine of the same step.
See ``ear_oracle.cpp`` for the definition each step follows (SVG-EAR, by
section).  ``pipeline`` runs the five steps in order for one head.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
from typing import Optional

import numpy as np

from . import build as _build

_LIB = None
_f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(np.int64, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32


def lib():
    global _LIB
    if _LIB is None:
        L = ctypes.CDLL(_build.build())
        L.oracle_kmeans.argtypes = [_f64p, _i64, _i32, _i32, _i32, _f64p, _f64p, _i32p, _i64p]
        L.oracle_permute.argtypes = [_i32p, _i64, _i32, _i32p, _i64p]
        L.oracle_segment_mean.argtypes = [_f64p, _i32p, _i64, _i32, _i32, _f64p]
        L.oracle_probe.argtypes = [_f64p, _i64p, _f64p, _i32p, _f64p, _i64p, _i64, _i32, _i32,
                                   _i32, ctypes.c_double, _f64p]
        L.oracle_probe_weights.argtypes = [_f64p, _i64p, _f64p, _i32p, _f64p, _i64p, _f64p,
                                           _f64p, _i64, _i32, _i32, _i32, ctypes.c_double,
                                           _i32, _f64p]
        L.oracle_route.argtypes = [_f64p, _i64p, _i64p, _i32, _i32, _i64, _i64, ctypes.c_double,
                                   _i32, _u8p, ctypes.POINTER(ctypes.c_int64)]
        L.oracle_attention.argtypes = [_f64p, _f64p, _f64p, _i32p, _i32p, _f64p, _f64p, _i64p,
                                       _u8p, _i64, _i64, _i32, _i32, _i32, ctypes.c_double,
                                       _i32, _f64p, _f64p]
        L.oracle_cluster_stats.argtypes = [_f64p, _i32p, _f64p, _i64, _i32,
                                           ctypes.POINTER(ctypes.c_double),
                                           ctypes.POINTER(ctypes.c_double)]
        L.oracle_cluster_stats.restype = None
        L.oracle_normalizer_change.argtypes = [_f64p, _f64p, _i64]
        L.oracle_normalizer_change.restype = ctypes.c_double
        L.oracle_route_rows.argtypes = [_f64p, _i64p, _i64p, _i32, _i32, _i64p, _u8p, _i64p]
        L.oracle_route_rows.restype = None
        L.oracle_topp_budget.argtypes = [_f64p, _i64p, _f64p, _i64p, _i32, _i32, _i32,
                                         ctypes.c_double, ctypes.c_double, _i64p]
        L.oracle_topp_budget.restype = None
        L.oracle_max_threads.restype = ctypes.c_int32
        for fn in (L.oracle_kmeans, L.oracle_permute, L.oracle_segment_mean, L.oracle_probe,
                   L.oracle_probe_weights, L.oracle_route, L.oracle_attention):
            fn.restype = None
        _LIB = L
    return _LIB


def _f64(x):
    return np.ascontiguousarray(x, dtype=np.float64)


def _ci32(x):
    return np.ascontiguousarray(x, dtype=np.int32)


def _ci64(x):
    return np.ascontiguousarray(x, dtype=np.int64)


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def kmeans(x, init, iters):
    """Lloyd k-means from ``init`` (SVG-EAR §4.1). Returns (centroids, labels, counts)."""
    x = _f64(x)
    init = _f64(init)
    n, d = x.shape
    c = init.shape[0]
    cent = np.empty((c, d), np.float64)
    labels = np.empty(n, np.int32)
    counts = np.empty(c, np.int64)
    lib().oracle_kmeans(x, n, d, c, int(iters), init, cent, labels, counts)
    return cent, labels, counts


def permute(labels, n_clusters):
    """Stable sort of token indices by label (SVG-EAR §3.1). Returns (perm, offsets)."""
    labels = _ci32(labels)
    perm = np.empty(labels.shape[0], np.int32)
    offsets = np.empty(n_clusters + 1, np.int64)
    lib().oracle_permute(labels, labels.shape[0], int(n_clusters), perm, offsets)
    return perm, offsets


def segment_mean(x, labels, n_clusters):
    """Per-cluster mean of the rows of x (SVG-EAR §4.3, v̄)."""
    x = _f64(x)
    out = np.empty((n_clusters, x.shape[1]), np.float64)
    lib().oracle_segment_mean(x, _ci32(labels), x.shape[0], x.shape[1], int(n_clusters), out)
    return out


def probe(q_cent, q_counts, k, k_labels, k_cent, k_counts, scale):
    """E[a, b] = sum_{j in b} (s q̄_a·k_j - s q̄_a·k̄_b)^2 (SVG-EAR §4.2)."""
    q_cent = _f64(q_cent)
    k = _f64(k)
    k_cent = _f64(k_cent)
    cq, d = q_cent.shape
    ck = k_cent.shape[0]
    e = np.empty((cq, ck), np.float64)
    lib().oracle_probe(q_cent, _ci64(q_counts), k, _ci32(k_labels), k_cent, _ci64(k_counts),
                       k.shape[0], d, cq, ck, float(scale), e)
    return e


PROBE_LOGIT, PROBE_WEIGHTS, PROBE_VALUE = 0, 1, 2


def probe_weights(q_cent, q_counts, k, k_labels, k_cent, k_counts, v, v_cent, scale, mode):
    """Error probes on the unnormalized attention weights (SVG-EAR §4.2 relaxed
    problem, §4.3 value-aware estimate, §4.4 running maximum): mode 1 sums
    (w_j - w̄_b)^2, mode 2 sums ||w_j v_j - w̄_b v̄_b||^2, with w = e^{z - m_a}."""
    q_cent = _f64(q_cent)
    k = _f64(k)
    k_cent = _f64(k_cent)
    cq, d = q_cent.shape
    ck = k_cent.shape[0]
    vv = _f64(v) if v is not None else np.zeros_like(k)
    vc = _f64(v_cent) if v_cent is not None else np.zeros_like(k_cent)
    e = np.empty((cq, ck), np.float64)
    lib().oracle_probe_weights(q_cent, _ci64(q_counts), k, _ci32(k_labels), k_cent,
                               _ci64(k_counts), vv, vc, k.shape[0], d, cq, ck, float(scale),
                               int(mode), e)
    return e


def route(e, q_counts, k_counts, n_q, n_k, density, mode=0):
    """Greedy error-to-cost routing under the density budget (SVG-EAR §4.2).

    Returns (exact uint8 [C_q, C_k], exact_pairs)."""
    e = _f64(e)
    cq, ck = e.shape
    exact = np.empty((cq, ck), np.uint8)
    pairs = ctypes.c_int64(0)
    lib().oracle_route(e, _ci64(q_counts), _ci64(k_counts), cq, ck, int(n_q), int(n_k),
                       float(density), int(mode), exact, ctypes.byref(pairs))
    return exact, int(pairs.value)


def block_lists(exact):
    """Per query cluster, the exact key clusters in ascending order (CSR)."""
    exact = np.asarray(exact)
    per = exact.astype(np.int64).sum(axis=1)
    offsets = np.zeros(exact.shape[0] + 1, np.int64)
    np.cumsum(per, out=offsets[1:])
    lst = np.nonzero(exact)[1].astype(np.int32)
    return offsets, lst


def attention(q, k, v, q_labels, k_labels, k_cent, v_cent, k_counts, exact, scale,
              compensate=True):
    """Block-sparse attention with linear compensation (SVG-EAR §4.1, §4.3).

    Returns (O [N_q, d] in original order, lse [N_q])."""
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    nq, d = q.shape
    nk = k.shape[0]
    exact = np.ascontiguousarray(exact, dtype=np.uint8)
    cq, ck = exact.shape
    o = np.empty((nq, d), np.float64)
    lse = np.empty(nq, np.float64)
    lib().oracle_attention(q, k, v, _ci32(q_labels), _ci32(k_labels), _f64(k_cent),
                           _f64(v_cent), _ci64(k_counts), exact, nq, nk, d, cq, ck,
                           float(scale), int(bool(compensate)), o, lse)
    return o, lse


@dataclasses.dataclass
class HeadResult:
    q_cent: np.ndarray
    q_labels: np.ndarray
    q_counts: np.ndarray
    k_cent: np.ndarray
    k_labels: np.ndarray
    k_counts: np.ndarray
    q_perm: np.ndarray
    q_offsets: np.ndarray
    k_perm: np.ndarray
    k_offsets: np.ndarray
    v_mean: np.ndarray
    e: np.ndarray
    exact: np.ndarray
    exact_pairs: int
    blk_offsets: np.ndarray
    blk_list: np.ndarray
    o: np.ndarray
    lse: np.ndarray


def pipeline(q, k, v, q_init, k_init, iters, density, mode=0, compensate=True,
             scale: Optional[float] = None) -> HeadResult:
    """All five steps for one head, in the order of SVG-EAR §3.1 / §4."""
    d = q.shape[1]
    s = 1.0 / math.sqrt(d) if scale is None else scale
    qc, ql, qn = kmeans(q, q_init, iters)
    kc, kl, kn = kmeans(k, k_init, iters)
    qp, qo = permute(ql, qc.shape[0])
    kp, ko = permute(kl, kc.shape[0])
    vm = segment_mean(v, kl, kc.shape[0])
    e = probe(qc, qn, k, kl, kc, kn, s)
    exact, pairs = route(e, qn, kn, q.shape[0], k.shape[0], density, mode)
    bo, bl = block_lists(exact)
    o, lse = attention(q, k, v, ql, kl, kc, vm, kn, exact, s, compensate)
    return HeadResult(qc, ql, qn, kc, kl, kn, qp, qo, kp, ko, vm, e, exact, pairs, bo, bl, o, lse)


def cluster_stats(x, labels, centroids):
    """(δ^2, K_max): mean squared row-to-centroid distance and largest row norm
    (SVG-EAR §4.2 bound residual, §5.3 "Effect of clustering")."""
    x = _f64(x)
    ms = ctypes.c_double(0.0)
    mx = ctypes.c_double(0.0)
    lib().oracle_cluster_stats(x, _ci32(labels), _f64(centroids), x.shape[0], x.shape[1],
                               ctypes.byref(ms), ctypes.byref(mx))
    return float(ms.value), float(mx.value)


def bound_residual(delta_sq, k_max, n_k, d):
    """The residual 8 δ_q^2 K_max^2 / (N_k d) of the SVG-EAR §4.2 bound."""
    return 8.0 * delta_sq * k_max ** 2 / (n_k * d)


def normalizer_change(lse_sparse, lse_dense):
    """Average |Z_sparse / Z_dense - 1| over queries, Z = e^{lse} (SVG-EAR §5.1)."""
    a = _f64(lse_sparse)
    b = _f64(lse_dense)
    return float(lib().oracle_normalizer_change(a, b, a.shape[0]))


def route_rows(e, q_counts, k_counts, row_budget):
    """Greedy error-to-cost routing inside each query cluster under its own
    budget (SVG-EAR §5 "Implementation"). Returns (exact [C_q, C_k], pairs [C_q])."""
    e = _f64(e)
    cq, ck = e.shape
    exact = np.empty((cq, ck), np.uint8)
    pairs = np.empty(cq, np.int64)
    lib().oracle_route_rows(e, _ci64(q_counts), _ci64(k_counts), cq, ck, _ci64(row_budget),
                            exact, pairs)
    return exact, pairs


def topp_budget(q_cent, q_counts, k_cent, k_counts, scale, p):
    """Per query cluster: |a| x keys of the smallest set of key clusters, by
    decreasing centroid attention mass, that reaches fraction p of it."""
    q_cent = _f64(q_cent)
    k_cent = _f64(k_cent)
    cq, d = q_cent.shape
    out = np.empty(cq, np.int64)
    lib().oracle_topp_budget(q_cent, _ci64(q_counts), k_cent, _ci64(k_counts), cq,
                             k_cent.shape[0], d, float(scale), float(p), out)
    return out


def uniform_row_budget(q_counts, n_k, density):
    """Each query cluster's share of the global budget: floor(rho |a| N_k)."""
    qn = np.asarray(q_counts, np.int64)
    return np.floor(density * (qn * int(n_k)).astype(np.float64)).astype(np.int64)
