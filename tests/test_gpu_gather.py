"""GPU parity of the gathered layer: the probe and the attention reading Q, K
and V in their original token order through the permutations (SVG-EAR §3.1's
cluster-contiguous layout folded into the loads; the attention fetches rows
with TMA tile::gather4).

Each gathered call is checked twice: bit for bit against the same call on
permuted copies (the smem tiles hold the same rows, and rows past a cluster
are masked on both paths), and against the fp64 oracle at the attention
tolerances of tests/parity_util.py.
"""
import math

import numpy as np
import pytest
import torch

import parity_util as pu
from clustered_block_sparse_b200 import ear
from clustered_block_sparse_b200 import inputs as gen
from oracle import ear_oracle as eo

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from clustered_block_sparse_b200 import build
    build.build()
    yield
    assert ear.ear_get_device_status() == 0


MID2 = gen.MID.with_(heads=2)
CONFIGS = {"tiny": gen.TINY, "mid": MID2,
           # many small key clusters: partial 32-row boxes, several clusters per chunk
           "small_k": gen.MID.with_(heads=2, n=2000, n_centres=60, c_q=7, c_k=400, iters=2,
                                    density=0.3),
           "d64": gen.MID.with_(heads=2, n=3001, d=64, c_q=13, c_k=77, iters=3, density=0.2)}


@pytest.fixture(scope="module")
def cases():
    out = {}
    for name, w in CONFIGS.items():
        L = gen.make_layer(w)
        runs = [eo.pipeline(L.q[h], L.k[h], L.v[h], L.q_init[h], L.k_init[h], w.iters, w.density)
                for h in range(len(L.heads))]
        out[name] = (L, runs)
    return out


def _stack(runs, attr, dtype=None):
    a = np.stack([getattr(r, attr) for r in runs])
    return a if dtype is None else a.astype(dtype)


def _blk_list(runs, c_q, c_k):
    return np.stack([np.pad(r.blk_list, (0, c_q * c_k - len(r.blk_list)))
                     for r in runs]).astype(np.int32)


def _attention_both(L, runs, compensate):
    """(O, lse) of ear_attention on permuted copies and of ear_attention_gather."""
    w = L.workload
    t = pu.torch_dtype(w.dtype)
    qp, kp = _stack(runs, "q_perm", np.int32), _stack(runs, "k_perm", np.int32)
    q, k, v = pu.dev(L.q, t), pu.dev(L.k, t), pu.dev(L.v, t)
    qpd, kpd = pu.dev(qp), pu.dev(kp)
    idx_q, idx_k = qpd.long()[..., None], kpd.long()[..., None]
    qx = torch.gather(q, 1, idx_q.expand(-1, -1, w.d)).contiguous()
    kx = torch.gather(k, 1, idx_k.expand(-1, -1, w.d)).contiguous()
    vx = torch.gather(v, 1, idx_k.expand(-1, -1, w.d)).contiguous()
    common = dict(q_offsets=pu.dev(_stack(runs, "q_offsets", np.int32)),
                  k_offsets=pu.dev(_stack(runs, "k_offsets", np.int32)), q_perm=qpd,
                  k_centroids=pu.dev(_stack(runs, "k_cent", np.float32)),
                  v_centroids=pu.dev(_stack(runs, "v_mean", np.float32)),
                  exact=pu.dev(np.ascontiguousarray(_stack(runs, "exact"))),
                  blk_offsets=pu.dev(_stack(runs, "blk_offsets", np.int32)),
                  blk_list=pu.dev(_blk_list(runs, w.c_q, w.c_k)), scale=pu.scale_of(w.d),
                  compensate=compensate, want_lse=True)
    o_p, lse_p = ear.ear_attention(qx, kx, vx, **common)
    o_g, lse_g = ear.ear_attention_gather(q, k, v, k_perm_idx=kpd, **common)
    return (pu.host(o_p), pu.host(lse_p)), (pu.host(o_g), pu.host(lse_g))


@pytest.mark.parametrize("cfg", list(CONFIGS))
@pytest.mark.parametrize("compensate", [True, False])
def test_attention_gather_is_the_permuted_attention(cases, cfg, compensate):
    L, runs = cases[cfg]
    w = L.workload
    (o_p, lse_p), (o_g, lse_g) = _attention_both(L, runs, compensate)
    np.testing.assert_array_equal(o_g, o_p)
    np.testing.assert_array_equal(lse_g, lse_p)
    for h, r in enumerate(runs):
        o_ref, lse_ref = eo.attention(L.q[h], L.k[h], L.v[h], r.q_labels, r.k_labels, r.k_cent,
                                      r.v_mean, r.k_counts, r.exact, pu.scale_of(w.d), compensate)
        ok = np.isfinite(lse_ref)
        pu.assert_attention_close(o_g[h][ok], o_ref[ok], w.dtype)
        np.testing.assert_allclose(lse_g[h][ok], lse_ref[ok], rtol=0, atol=pu.LSE_TOL[w.dtype])


@pytest.mark.parametrize("compensate", [True, False])
def test_attention_gather_ragged_clusters_and_lengths(compensate):
    """N_q != N_k, cluster sizes that are not multiples of 4 or 32 (every box
    and Q tile ends in repeated rows), one query cluster of 1 row, empty key
    clusters, and key lists beyond the 2,048 entries staged in shared memory."""
    rng = np.random.default_rng(2024)
    d = 128
    q_sizes = np.array([1, 257, 3, 130, 0, 77])
    k_sizes = rng.integers(0, 5, 2100)
    k_sizes[:10] = [33, 0, 1, 65, 31, 0, 2, 97, 5, 4]
    nq, nk = int(q_sizes.sum()), int(k_sizes.sum())
    q = gen.round_to_bf16(rng.standard_normal((nq, d)))
    k = gen.round_to_bf16(rng.standard_normal((nk, d)))
    v = gen.round_to_bf16(rng.standard_normal((nk, d)))
    ql = np.repeat(np.arange(len(q_sizes)), q_sizes).astype(np.int32)
    kl = np.repeat(np.arange(len(k_sizes)), k_sizes).astype(np.int32)
    # tokens in a shuffled original order; perm[r] = original index of permuted row r
    q_perm = rng.permutation(nq).astype(np.int32)
    k_perm = rng.permutation(nk).astype(np.int32)
    q_orig = np.empty_like(q)
    q_orig[q_perm] = q
    k_orig = np.empty_like(k)
    k_orig[k_perm] = k
    v_orig = np.empty_like(v)
    v_orig[k_perm] = v
    ql_orig = np.empty_like(ql)
    ql_orig[q_perm] = ql
    kl_orig = np.empty_like(kl)
    kl_orig[k_perm] = kl
    exact = (rng.random((len(q_sizes), len(k_sizes))) < 0.6).astype(np.uint8)
    exact[0] = 1                                      # a list of 2,100 clusters
    kc = eo.segment_mean(k, kl, len(k_sizes)).astype(np.float32)
    vm = eo.segment_mean(v, kl, len(k_sizes)).astype(np.float32)
    qo = np.concatenate([[0], np.cumsum(q_sizes)]).astype(np.int32)
    ko = np.concatenate([[0], np.cumsum(k_sizes)]).astype(np.int32)
    o_lists, l_lists = eo.block_lists(exact)
    bl = np.zeros(exact.size, np.int32)
    bl[:len(l_lists)] = l_lists
    s = pu.scale_of(d)
    t = torch.bfloat16
    o, lse = ear.ear_attention_gather(
        pu.dev(q_orig[None], t), pu.dev(k_orig[None], t), pu.dev(v_orig[None], t),
        pu.dev(qo[None]), pu.dev(ko[None]), pu.dev(q_perm[None]), pu.dev(k_perm[None]),
        pu.dev(kc[None]), pu.dev(vm[None]), pu.dev(exact[None]),
        pu.dev(o_lists[None].astype(np.int32)), pu.dev(bl[None]), s, compensate, want_lse=True)
    o, lse = pu.host(o)[0], pu.host(lse)[0]
    o_ref, lse_ref = eo.attention(q_orig, k_orig, v_orig, ql_orig, kl_orig, kc, vm,
                                  k_sizes.astype(np.int64), exact, s, compensate)
    ok = np.isfinite(lse_ref)
    pu.assert_attention_close(o[ok], o_ref[ok], "bf16")
    np.testing.assert_allclose(lse[ok], lse_ref[ok], rtol=0, atol=pu.LSE_TOL["bf16"])
    assert np.all(o[~ok] == 0) and np.all(np.isneginf(lse[~ok]))


@pytest.mark.parametrize("cfg", list(CONFIGS))
def test_probe_gather_is_the_permuted_probe(cases, cfg):
    L, runs = cases[cfg]
    w = L.workload
    t = pu.torch_dtype(w.dtype)
    k, v = pu.dev(L.k, t), pu.dev(L.v, t)
    kpd = pu.dev(_stack(runs, "k_perm", np.int32))
    idx = kpd.long()[..., None].expand(-1, -1, w.d)
    kx = torch.gather(k, 1, idx).contiguous()
    vx = torch.gather(v, 1, idx).contiguous()
    qc = pu.dev(_stack(runs, "q_cent", np.float32))
    qn = pu.dev(_stack(runs, "q_counts", np.int32))
    kc = pu.dev(_stack(runs, "k_cent", np.float32))
    ko = pu.dev(_stack(runs, "k_offsets", np.int32))
    vm = pu.dev(_stack(runs, "v_mean", np.float32))
    modes = [0] if w.dtype == "f32" else [0, 1, 2]
    for mode in modes:
        e_p = ear.ear_probe(qc, qn, kc, kx, ko, mode=mode, v_perm=vx, v_centroids=vm)
        e_g = ear.ear_probe_gather(qc, qn, kc, k, kpd, ko, mode=mode, v=v, v_centroids=vm)
        np.testing.assert_array_equal(pu.host(e_g), pu.host(e_p))
    e_g = pu.host(ear.ear_probe_gather(qc, qn, kc, k, kpd, ko))
    for h, r in enumerate(runs):
        np.testing.assert_allclose(e_g[h], r.e, rtol=2e-5, atol=1e-7 * r.e.max())


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_permute_apply_means_only(dtype, d):
    rng = np.random.default_rng(8)
    bh, n, c = 2, 5000, 37
    x = gen.round_to_dtype(rng.standard_normal((bh, n, d)), dtype)
    lab = rng.integers(0, c, (bh, n)).astype(np.int32)
    t = pu.torch_dtype(dtype)
    perm, offs, _, _ = ear.ear_permute(pu.dev(lab), c)
    xd = pu.dev(x, t)
    xp, m_full = ear.ear_permute_apply(perm, offs, xd, seg_mean=True)
    none, m_only = ear.ear_permute_apply(perm, offs, xd, seg_mean=True, write_perm=False)
    assert none is None
    np.testing.assert_array_equal(pu.host(m_only), pu.host(m_full))
    for h in range(bh):
        ref = eo.segment_mean(x[h], lab[h], c)
        np.testing.assert_allclose(pu.host(m_only)[h], ref, rtol=1e-6, atol=1e-6)


def _rest_of_layer(q, k, v, km, w, gather):
    """Permute, probe, route and attention after a given k-means (the k-means
    centroid sums use float atomics, so two k-means runs may differ in the last
    bits; both layouts start from the same clustering)."""
    (qc, ql, qn), (kc, kl, kn) = km
    n = q.shape[1]
    if gather:
        qp, qo, _, _ = ear.ear_permute(ql, w.c_q)
        kp, ko, _, _ = ear.ear_permute(kl, w.c_k)
        _, vm = ear.ear_permute_apply(kp, ko, v, seg_mean=True, write_perm=False)
        e = ear.ear_probe_gather(qc, qn, kc, k, kp, ko)
    else:
        qp, qo, qx, _ = ear.ear_permute(ql, w.c_q, q)
        kp, ko, kx, _ = ear.ear_permute(kl, w.c_k, k)
        vx, vm = ear.ear_permute_apply(kp, ko, v, seg_mean=True)
        e = ear.ear_probe(qc, qn, kc, kx, ko)
    exact, bo, bl, pairs = ear.ear_route(e, qn, kn, n, n, w.density)
    if gather:
        o, lse = ear.ear_attention_gather(q, k, v, qo, ko, qp, kp, kc, vm, exact, bo, bl,
                                          want_lse=True)
    else:
        o, lse = ear.ear_attention(qx, kx, vx, qo, ko, qp, kc, vm, exact, bo, bl, want_lse=True)
    return {"o": o, "lse": lse, "e": e, "exact": exact, "blk_offsets": bo, "blk_list": bl,
            "exact_pairs": pairs, "v_mean": vm, "q_perm": qp, "k_perm": kp}


@pytest.mark.parametrize("cfg", list(CONFIGS))
def test_layer_gathered_equals_layer_permuted(cases, cfg):
    L, _ = cases[cfg]
    w = L.workload
    t = pu.torch_dtype(w.dtype)
    q, k, v = pu.dev(L.q, t), pu.dev(L.k, t), pu.dev(L.v, t)
    km = (ear.ear_kmeans(q, pu.dev(L.q_init), w.iters), ear.ear_kmeans(k, pu.dev(L.k_init), w.iters))
    a = _rest_of_layer(q, k, v, km, w, False)
    b = _rest_of_layer(q, k, v, km, w, True)
    for name, x in a.items():
        if name != "blk_list":
            np.testing.assert_array_equal(pu.host(b[name]), pu.host(x), name)
    # block lists: the entries ear_route wrote (the rest of the buffer is scratch)
    bo = pu.host(a["blk_offsets"])
    for h in range(bo.shape[0]):
        n = bo[h, -1]
        np.testing.assert_array_equal(pu.host(b["blk_list"])[h, :n], pu.host(a["blk_list"])[h, :n])
    # and the public layer call takes the gathered path end to end
    res = ear.ear_layer(q, k, v, pu.dev(L.q_init), pu.dev(L.k_init), w.iters, w.density,
                        gather=True)
    assert torch.isfinite(res.o.float()).all()


@pytest.mark.slow
def test_wan_layer_gathered_full_size():
    """The 40-head Wan2.x layer through the gathered path: every output equals
    the permuted path's bit for bit, and sampled queries match the oracle given
    the layer's own mask, labels and centroids."""
    w = gen.WAN
    L = gen.make_layer(w)
    t = torch.bfloat16
    q, k, v = pu.dev(L.q, t), pu.dev(L.k, t), pu.dev(L.v, t)
    km = (ear.ear_kmeans(q, pu.dev(L.q_init), w.iters), ear.ear_kmeans(k, pu.dev(L.k_init), w.iters))
    a = _rest_of_layer(q, k, v, km, w, False)
    b = _rest_of_layer(q, k, v, km, w, True)
    torch.cuda.synchronize()
    assert ear.ear_get_device_status() == 0
    for name, x in a.items():
        if name != "blk_list":
            assert torch.equal(b[name], x), name
    s = pu.scale_of(w.d)
    rng = np.random.default_rng(3)
    o = pu.host(b["o"])
    for h in (0, w.heads - 1):
        qlab, klab = pu.host(km[0][1])[h], pu.host(km[1][1])[h]
        kc, kn = pu.host(km[1][0])[h], pu.host(km[1][2])[h]
        qi = rng.choice(w.n, 256, replace=False)
        vm = eo.segment_mean(L.v[h], klab, w.c_k)
        o_ref, _ = eo.attention(L.q[h][qi], L.k[h], L.v[h], qlab[qi], klab, kc, vm, kn,
                                pu.host(b["exact"])[h], s)
        pu.assert_attention_close(o[h][qi], o_ref, "bf16")
