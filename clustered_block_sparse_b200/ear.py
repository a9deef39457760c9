"""Python binding of libear: one function per C entry point, same names.

Argument marshalling only: every step runs in libear's CUDA kernels.  Tensors
are torch CUDA tensors (torch provides device memory and the stream); outputs
are allocated here when not passed in.  Errors raise ``EarError``.

Citations "SVG-EAR §x" are to "SVG-EAR: Parameter-Free Linear Compensation for
Sparse Video Generation via Error-aware Routing" (arXiv 2603.08982).
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
from typing import Optional

import torch

from . import _native as N
from ._native import EarError  # noqa: F401  (re-export)

_DT = {torch.float32: N.EAR_F32, torch.bfloat16: N.EAR_BF16}


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"unsupported dtype {t.dtype}; libear takes float32 or bfloat16")
    return _DT[t.dtype]


def _need(t: torch.Tensor, name: str):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


def _workspace(op, bh, n_q, n_k, d, c_q, c_k, device):
    nbytes = N.workspace_bytes(op, bh, n_q, n_k, d, c_q, c_k)
    if nbytes == 0:
        return None, 0
    return torch.empty(nbytes, dtype=torch.uint8, device=device), nbytes


def ear_kmeans(x: torch.Tensor, init: torch.Tensor, iters: int):
    """Lloyd k-means (SVG-EAR §4.1). x [BH,N,d], init [BH,C,d] float32.

    Returns (centroids [BH,C,d] f32, labels [BH,N] i32, counts [BH,C] i32)."""
    _need(x, "x")
    _need(init, "init")
    bh, n, d = x.shape
    c = init.shape[1]
    cent = torch.empty((bh, c, d), dtype=torch.float32, device=x.device)
    labels = torch.empty((bh, n), dtype=torch.int32, device=x.device)
    counts = torch.empty((bh, c), dtype=torch.int32, device=x.device)
    ws, nb = _workspace(N.EAR_OP_KMEANS, bh, n, 0, d, c, 0, x.device)
    N.check("ear_kmeans", N.lib().ear_kmeans(
        _p(x), _dtype(x), bh, n, d, c, int(iters), _p(init), _p(cent), _p(labels), _p(counts),
        _p(ws), nb, _stream(x.device)))
    return cent, labels, counts


_SIDE_STREAMS = {}


def _side_stream(device) -> torch.cuda.Stream:
    dev = torch.device(device)
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    if key not in _SIDE_STREAMS:
        _SIDE_STREAMS[key] = torch.cuda.Stream(device=dev)
    return _SIDE_STREAMS[key]


def ear_kmeans_pair(q, q_init, k, k_init, iters: int, streams: int = 2, q_after=None):
    """Q's and K's k-means (independent of each other, SVG-EAR §4.1).  With
    streams=2, K's runs on a side stream beside Q's on the current stream and
    the current stream waits for it before returning: each call's kernels fill
    the other's tails and small launches.  q_after(qc, ql, qn), if given, runs
    on the current stream right after Q's k-means (under K's, which takes
    longer); its result is returned third.
    Returns ((qc, ql, qn), (kc, kl, kn), q_after's result or None)."""
    if streams == 1:
        qres = ear_kmeans(q, q_init, iters)
        kres = ear_kmeans(k, k_init, iters)
        return qres, kres, (q_after(*qres) if q_after is not None else None)
    cur = torch.cuda.current_stream(q.device)
    side = _side_stream(q.device)
    side.wait_stream(cur)
    with torch.cuda.stream(side):
        kres = ear_kmeans(k, k_init, iters)
    qres = ear_kmeans(q, q_init, iters)
    extra = q_after(*qres) if q_after is not None else None
    cur.wait_stream(side)
    for t in kres:
        t.record_stream(cur)  # allocated on the side stream, used on this one
    return qres, kres, extra


def ear_permute(labels: torch.Tensor, n_clusters: int, x: Optional[torch.Tensor] = None,
                seg_mean: bool = False):
    """Stable cluster-contiguous permutation (SVG-EAR §3.1).

    Returns (perm [BH,N] i32, offsets [BH,C+1] i32, x_perm or None, mean [BH,C,d] f32 or None)."""
    _need(labels, "labels")
    bh, n = labels.shape
    dev = labels.device
    perm = torch.empty((bh, n), dtype=torch.int32, device=dev)
    offsets = torch.empty((bh, n_clusters + 1), dtype=torch.int32, device=dev)
    x_perm = mean = None
    d, dt = 0, 0
    if x is not None:
        _need(x, "x")
        d, dt = x.shape[2], _dtype(x)
        x_perm = torch.empty_like(x)
        if seg_mean:
            mean = torch.empty((bh, n_clusters, d), dtype=torch.float32, device=dev)
    ws, nb = _workspace(N.EAR_OP_PERMUTE, bh, n, 0, d, n_clusters, 0, dev)
    N.check("ear_permute", N.lib().ear_permute(
        _p(labels), bh, n, n_clusters, _p(perm), _p(offsets), _p(x), _p(x_perm), dt, d, _p(mean),
        _p(ws), nb, _stream(dev)))
    return perm, offsets, x_perm, mean


def ear_permute_apply(perm: torch.Tensor, offsets: torch.Tensor, x: torch.Tensor,
                      seg_mean: bool = False, write_perm: bool = True):
    """X_perm[r] = X[perm[r]] with a permutation made by ear_permute, plus the
    optional per-cluster means (SVG-EAR §4.3: V in K's cluster order, v̄).
    write_perm=False (with seg_mean) computes the means alone.

    Returns (x_perm or None, mean [BH,C,d] f32 or None)."""
    for t, nm in ((perm, "perm"), (offsets, "offsets"), (x, "x")):
        _need(t, nm)
    bh, n, d = x.shape
    c = offsets.shape[1] - 1
    x_perm = torch.empty_like(x) if write_perm else None
    mean = torch.empty((bh, c, d), dtype=torch.float32, device=x.device) if seg_mean else None
    N.check("ear_permute_apply", N.lib().ear_permute_apply(
        _p(perm), _p(offsets), bh, n, c, _p(x), _p(x_perm), _dtype(x), d, _p(mean),
        _stream(x.device)))
    return x_perm, mean


def ear_permute_static(labels: torch.Tensor, n_clusters: int, x: Optional[torch.Tensor] = None,
                       seg_mean: bool = False):
    """ear_permute without a workspace, for callers that cannot allocate device
    memory: the scratch lives in a fixed array inside libear (at most
    EAR_PERMUTE_STATIC_MAX_BYTES).  Same results as ear_permute.  Calls that
    overlap on the GPU share that array and race; run them one at a time."""
    _need(labels, "labels")
    bh, n = labels.shape
    dev = labels.device
    perm = torch.empty((bh, n), dtype=torch.int32, device=dev)
    offsets = torch.empty((bh, n_clusters + 1), dtype=torch.int32, device=dev)
    x_perm = mean = None
    d, dt = 0, 0
    if x is not None:
        _need(x, "x")
        d, dt = x.shape[2], _dtype(x)
        x_perm = torch.empty_like(x)
        if seg_mean:
            mean = torch.empty((bh, n_clusters, d), dtype=torch.float32, device=dev)
    N.check("ear_permute_static", N.lib().ear_permute_static(
        _p(labels), bh, n, n_clusters, _p(perm), _p(offsets), _p(x), _p(x_perm), dt, d, _p(mean),
        _stream(dev)))
    return perm, offsets, x_perm, mean


def ear_probe(q_centroids, q_counts, k_centroids, k_perm, k_offsets, scale: Optional[float] = None,
              mode: int = 0, v_perm=None, v_centroids=None):
    """Per-block compensation-error estimate (SVG-EAR §4.2), E [BH,C_q,C_k] f32.

    mode 0: E[a,b] = sum_{j in b} (s q̄_a·k_j - s q̄_a·k̄_b)^2; mode 1: the same on the
    unnormalized weights e^{z - m_a}; mode 2: value-aware (needs v_perm, v_centroids)."""
    for t, nm in ((q_centroids, "q_centroids"), (q_counts, "q_counts"), (k_centroids, "k_centroids"),
                  (k_perm, "k_perm"), (k_offsets, "k_offsets")):
        _need(t, nm)
    if mode == N.EAR_PROBE_VALUE:
        _need(v_perm, "v_perm")
        _need(v_centroids, "v_centroids")
    bh, c_q, d = q_centroids.shape
    c_k = k_centroids.shape[1]
    n_k = k_perm.shape[1]
    s = 1.0 / math.sqrt(d) if scale is None else scale
    e = torch.empty((bh, c_q, c_k), dtype=torch.float32, device=k_perm.device)
    ws, nb = _workspace(N.EAR_OP_PROBE, bh, 0, n_k, d, c_q, c_k, k_perm.device)
    N.check("ear_probe", N.lib().ear_probe(
        _p(q_centroids), _p(q_counts), _p(k_centroids), _p(k_perm), _dtype(k_perm), _p(k_offsets),
        bh, n_k, d, c_q, c_k, ctypes.c_float(s), int(mode), _p(v_perm), _p(v_centroids), _p(e),
        _p(ws), nb, _stream(k_perm.device)))
    return e


def ear_probe_gather(q_centroids, q_counts, k_centroids, k, k_perm_idx, k_offsets,
                     scale: Optional[float] = None, mode: int = 0, v=None, v_centroids=None):
    """ear_probe on keys (and values) in their original order: permuted key r is
    k[k_perm_idx[r]].  Same E as ear_probe(..., k[k_perm_idx], ...)."""
    for t, nm in ((q_centroids, "q_centroids"), (q_counts, "q_counts"), (k_centroids, "k_centroids"),
                  (k, "k"), (k_perm_idx, "k_perm_idx"), (k_offsets, "k_offsets")):
        _need(t, nm)
    if mode == N.EAR_PROBE_VALUE:
        _need(v, "v")
        _need(v_centroids, "v_centroids")
    bh, c_q, d = q_centroids.shape
    c_k = k_centroids.shape[1]
    n_k = k.shape[1]
    s = 1.0 / math.sqrt(d) if scale is None else scale
    e = torch.empty((bh, c_q, c_k), dtype=torch.float32, device=k.device)
    ws, nb = _workspace(N.EAR_OP_PROBE, bh, 0, n_k, d, c_q, c_k, k.device)
    N.check("ear_probe_gather", N.lib().ear_probe_gather(
        _p(q_centroids), _p(q_counts), _p(k_centroids), _p(k), _p(k_perm_idx), _dtype(k),
        _p(k_offsets), bh, n_k, d, c_q, c_k, ctypes.c_float(s), int(mode), _p(v), _p(v_centroids),
        _p(e), _p(ws), nb, _stream(k.device)))
    return e


def ear_route(e, q_counts, k_counts, n_q: int, n_k: int, density: float, ratio_mode: int = 0):
    """Greedy error-to-cost routing under the density budget (SVG-EAR §4.2).

    Returns (exact [BH,C_q,C_k] u8, blk_offsets [BH,C_q+1] i32, blk_list [BH,C_q*C_k] i32,
    exact_pairs [BH] i64)."""
    _need(e, "E")
    bh, c_q, c_k = e.shape
    dev = e.device
    exact = torch.empty((bh, c_q, c_k), dtype=torch.uint8, device=dev)
    blk_off = torch.empty((bh, c_q + 1), dtype=torch.int32, device=dev)
    blk_list = torch.empty((bh, c_q * c_k), dtype=torch.int32, device=dev)
    pairs = torch.empty((bh,), dtype=torch.int64, device=dev)
    ws, nb = _workspace(N.EAR_OP_ROUTE, bh, n_q, n_k, 0, c_q, c_k, dev)
    N.check("ear_route", N.lib().ear_route(
        _p(e), _p(q_counts), _p(k_counts), bh, n_q, n_k, c_q, c_k, ctypes.c_double(density),
        int(ratio_mode), _p(exact), _p(blk_off), _p(blk_list), _p(pairs), _p(ws), nb, _stream(dev)))
    return exact, blk_off, blk_list, pairs


def ear_route_rows(e, q_counts, k_counts, row_budget):
    """Greedy error-to-cost routing inside each query cluster under its own budget
    (SVG-EAR §5 "Implementation"). row_budget [BH,C_q] int64.

    Returns (exact [BH,C_q,C_k] u8, blk_offsets [BH,C_q+1] i32, blk_list [BH,C_q*C_k] i32,
    exact_pairs [BH] i64)."""
    for t, nm in ((e, "E"), (q_counts, "q_counts"), (k_counts, "k_counts"),
                  (row_budget, "row_budget")):
        _need(t, nm)
    bh, c_q, c_k = e.shape
    dev = e.device
    exact = torch.empty((bh, c_q, c_k), dtype=torch.uint8, device=dev)
    blk_off = torch.empty((bh, c_q + 1), dtype=torch.int32, device=dev)
    blk_list = torch.empty((bh, c_q * c_k), dtype=torch.int32, device=dev)
    pairs = torch.empty((bh,), dtype=torch.int64, device=dev)
    ws, nb = _workspace(N.EAR_OP_ROUTE_ROWS, bh, 0, 0, 0, c_q, c_k, dev)
    N.check("ear_route_rows", N.lib().ear_route_rows(
        _p(e), _p(q_counts), _p(k_counts), bh, c_q, c_k, _p(row_budget), _p(exact), _p(blk_off),
        _p(blk_list), _p(pairs), _p(ws), nb, _stream(dev)))
    return exact, blk_off, blk_list, pairs


def ear_topp_budget(q_centroids, q_counts, k_centroids, k_counts, p: float,
                    scale: Optional[float] = None):
    """SVG2-style adaptive per-query-cluster budgets from the centroid attention
    mass (top-p). Returns row_budget [BH,C_q] int64."""
    for t, nm in ((q_centroids, "q_centroids"), (q_counts, "q_counts"),
                  (k_centroids, "k_centroids"), (k_counts, "k_counts")):
        _need(t, nm)
    bh, c_q, d = q_centroids.shape
    c_k = k_centroids.shape[1]
    s = 1.0 / math.sqrt(d) if scale is None else scale
    out = torch.empty((bh, c_q), dtype=torch.int64, device=q_centroids.device)
    N.check("ear_topp_budget", N.lib().ear_topp_budget(
        _p(q_centroids), _p(q_counts), _p(k_centroids), _p(k_counts), bh, d, c_q, c_k,
        ctypes.c_float(s), ctypes.c_double(p), _p(out), _stream(q_centroids.device)))
    return out


def ear_uniform_budget(q_counts, n_k: int, density: float):
    """Each query cluster's share floor(rho |a| N_k) of the global budget. [BH,C_q] int64."""
    _need(q_counts, "q_counts")
    bh, c_q = q_counts.shape
    out = torch.empty((bh, c_q), dtype=torch.int64, device=q_counts.device)
    N.check("ear_uniform_budget", N.lib().ear_uniform_budget(
        _p(q_counts), bh, c_q, int(n_k), ctypes.c_double(density), _p(out),
        _stream(q_counts.device)))
    return out


def ear_cluster_stats(x: torch.Tensor, labels: torch.Tensor, centroids: torch.Tensor):
    """(δ^2 [BH] f64, max row norm [BH] f64): mean squared row-to-centroid distance
    and largest row norm (SVG-EAR §4.2 bound residual, §5.3)."""
    for t, nm in ((x, "x"), (labels, "labels"), (centroids, "centroids")):
        _need(t, nm)
    bh, n, d = x.shape
    c = centroids.shape[1]
    ms = torch.empty((bh,), dtype=torch.float64, device=x.device)
    mx = torch.empty((bh,), dtype=torch.float64, device=x.device)
    N.check("ear_cluster_stats", N.lib().ear_cluster_stats(
        _p(x), _dtype(x), _p(labels), _p(centroids), bh, n, d, c, _p(ms), _p(mx),
        _stream(x.device)))
    return ms, mx


def bound_residual(delta_sq, k_max, n_k: int, d: int):
    """The residual 8 δ_q^2 K_max^2 / (N_k d) of the SVG-EAR §4.2 bound."""
    return 8.0 * delta_sq * k_max ** 2 / (n_k * d)


def ear_normalizer_change(lse_sparse: torch.Tensor, lse_dense: torch.Tensor):
    """Per slice, mean |e^{lse_sparse - lse_dense} - 1| (SVG-EAR §5.1). [BH] f64."""
    _need(lse_sparse, "lse_sparse")
    _need(lse_dense, "lse_dense")
    bh, n = lse_sparse.shape
    out = torch.empty((bh,), dtype=torch.float64, device=lse_sparse.device)
    N.check("ear_normalizer_change", N.lib().ear_normalizer_change(
        _p(lse_sparse), _p(lse_dense), bh, n, _p(out), _stream(lse_sparse.device)))
    return out


def ear_attention(q_perm_x, k_perm_x, v_perm_x, q_offsets, k_offsets, q_perm, k_centroids,
                  v_centroids, exact, blk_offsets, blk_list, scale: Optional[float] = None,
                  compensate: bool = True, want_lse: bool = False, out: Optional[torch.Tensor] = None):
    """Block-sparse attention with linear compensation (SVG-EAR §4.1, §4.3).

    Returns (O [BH,N_q,d] in original query order, lse [BH,N_q] f32 or None)."""
    bh, n_q, d = q_perm_x.shape
    n_k = k_perm_x.shape[1]
    c_q = q_offsets.shape[1] - 1
    c_k = k_offsets.shape[1] - 1
    dev = q_perm_x.device
    s = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q_perm_x) if out is None else out
    lse = torch.empty((bh, n_q), dtype=torch.float32, device=dev) if want_lse else None
    ws, nb = _workspace(N.EAR_OP_ATTENTION, bh, n_q, n_k, d, c_q, c_k, dev)
    N.check("ear_attention", N.lib().ear_attention(
        _p(q_perm_x), _p(k_perm_x), _p(v_perm_x), _dtype(q_perm_x), _p(q_offsets), _p(k_offsets),
        _p(q_perm), _p(k_centroids), _p(v_centroids), _p(exact), _p(blk_offsets), _p(blk_list),
        bh, n_q, n_k, d, c_q, c_k, ctypes.c_float(s), N.EAR_COMPENSATE if compensate else 0,
        _p(o), _p(lse), _p(ws), nb, _stream(dev)))
    return o, lse


def ear_attention_gather(q, k, v, q_offsets, k_offsets, q_perm, k_perm_idx, k_centroids,
                         v_centroids, exact, blk_offsets, blk_list, scale: Optional[float] = None,
                         compensate: bool = True, want_lse: bool = False,
                         out: Optional[torch.Tensor] = None):
    """ear_attention on q, k, v in their original order (the permutation folded
    into the loads): permuted query r is q[q_perm[r]], permuted key r is
    k[k_perm_idx[r]] / v[k_perm_idx[r]].  Same O and lse as ear_attention on the
    permuted copies."""
    bh, n_q, d = q.shape
    n_k = k.shape[1]
    c_q = q_offsets.shape[1] - 1
    c_k = k_offsets.shape[1] - 1
    dev = q.device
    s = 1.0 / math.sqrt(d) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    lse = torch.empty((bh, n_q), dtype=torch.float32, device=dev) if want_lse else None
    ws, nb = _workspace(N.EAR_OP_ATTENTION, bh, n_q, n_k, d, c_q, c_k, dev)
    N.check("ear_attention_gather", N.lib().ear_attention_gather(
        _p(q), _p(k), _p(v), _dtype(q), _p(q_offsets), _p(k_offsets), _p(q_perm), _p(k_perm_idx),
        _p(k_centroids), _p(v_centroids), _p(exact), _p(blk_offsets), _p(blk_list),
        bh, n_q, n_k, d, c_q, c_k, ctypes.c_float(s), N.EAR_COMPENSATE if compensate else 0,
        _p(o), _p(lse), _p(ws), nb, _stream(dev)))
    return o, lse


def ear_selftest_wait_timeout(device=None) -> None:
    """Enqueue the bounded-wait self-test: the next ear_get_device_status() on
    this device reports EAR_ERR_TIMEOUT (after about one second)."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    N.check("ear_selftest_wait_timeout", N.lib().ear_selftest_wait_timeout(_stream(dev)))


def ear_get_device_status(device=None) -> int:
    """Synchronize the current stream and return (and clear) the latched device status."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    out = ctypes.c_int32(0)
    N.check("ear_get_device_status", N.lib().ear_get_device_status(ctypes.byref(out), _stream(dev)))
    return int(out.value)


@dataclasses.dataclass
class LayerResult:
    o: torch.Tensor
    lse: Optional[torch.Tensor]
    q_centroids: torch.Tensor
    q_labels: torch.Tensor
    q_counts: torch.Tensor
    k_centroids: torch.Tensor
    k_labels: torch.Tensor
    k_counts: torch.Tensor
    q_perm: torch.Tensor
    q_offsets: torch.Tensor
    k_perm: torch.Tensor
    k_offsets: torch.Tensor
    v_mean: torch.Tensor
    e: torch.Tensor
    exact: torch.Tensor
    blk_offsets: torch.Tensor
    blk_list: torch.Tensor
    exact_pairs: torch.Tensor


def ear_layer(q, k, v, q_init, k_init, iters: int, density: float, ratio_mode: int = 0,
              compensate: bool = True, want_lse: bool = False, scale: Optional[float] = None,
              out: Optional[torch.Tensor] = None, gather: bool = False) -> LayerResult:
    """One SVG-EAR attention layer: the five entry points in order (SVG-EAR §3.1, §4).

    gather=True keeps Q, K and V in their original order: the permutations are
    computed but never applied to a copy; the probe and the attention read rows
    through them (same results)."""
    n_q, n_k = q.shape[1], k.shape[1]
    # Q's permutation runs under K's k-means
    q_perm = (lambda qc_, ql_, qn_: ear_permute(ql_, q_init.shape[1], None if gather else q))
    (qc, ql, qn), (kc, kl, kn), (qp, qo, qx, _) = ear_kmeans_pair(q, q_init, k, k_init, iters,
                                                                  q_after=q_perm)
    if gather:
        kp, ko, _, _ = ear_permute(kl, k_init.shape[1])
        _, vm = ear_permute_apply(kp, ko, v, seg_mean=True, write_perm=False)
        e = ear_probe_gather(qc, qn, kc, k, kp, ko, scale)
    else:
        kp, ko, kx, _ = ear_permute(kl, k_init.shape[1], k)
        vx, vm = ear_permute_apply(kp, ko, v, seg_mean=True)
        e = ear_probe(qc, qn, kc, kx, ko, scale)
    exact, bo, bl, pairs = ear_route(e, qn, kn, n_q, n_k, density, ratio_mode)
    if gather:
        o, lse = ear_attention_gather(q, k, v, qo, ko, qp, kp, kc, vm, exact, bo, bl, scale,
                                      compensate, want_lse, out)
    else:
        o, lse = ear_attention(qx, kx, vx, qo, ko, qp, kc, vm, exact, bo, bl, scale, compensate,
                               want_lse, out)
    return LayerResult(o, lse, qc, ql, qn, kc, kl, kn, qp, qo, kp, ko, vm, e, exact, bo, bl, pairs)
