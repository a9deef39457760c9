"""GPU parity: every libear entry point against the fp64 CPU oracle on the
same seeded inputs, step by step (each step given the oracle's inputs to it),
end to end, on edge cases, and on sampled outputs at the Wan2.x layer size.

Tolerances (tests/parity_util.py): labels, permutations and routed blocks
bit-exact (a differing label/block only at a 1e-6 relative tie); attention
max-abs 2e-2 and rel-L2 5e-3 for bf16 inputs, max-abs 1e-4 for fp32.
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


def _tdt(w):
    return pu.torch_dtype(w.dtype)


MID2 = gen.MID.with_(heads=2)
CONFIGS = {"tiny": gen.TINY, "mid": MID2}


@pytest.fixture(scope="module")
def layers():
    return {k: gen.make_layer(w) for k, w in CONFIGS.items()}


@pytest.fixture(scope="module")
def oracle_runs(layers):
    out = {}
    for k, w in CONFIGS.items():
        L = layers[k]
        out[k] = [eo.pipeline(L.q[h], L.k[h], L.v[h], L.q_init[h], L.k_init[h], w.iters, w.density)
                  for h in range(len(L.heads))]
    return out


# --------------------------------------------------------------------------- k-means
@pytest.mark.parametrize("cfg", ["tiny", "mid"])
@pytest.mark.parametrize("which", ["q", "k"])
def test_kmeans_one_iteration_is_exact_argmin(layers, cfg, which):
    L = layers[cfg]
    x = getattr(L, which)
    init = L.q_init if which == "q" else L.k_init
    cent, lab, cnt = ear.ear_kmeans(pu.dev(x, _tdt(L.workload)), pu.dev(init), 1)
    cent, lab, cnt = pu.host(cent), pu.host(lab), pu.host(cnt)
    for h in range(x.shape[0]):
        c_ref, l_ref, n_ref = eo.kmeans(x[h], init[h], 1)
        nbad = pu.assert_labels_exact_or_tie(x[h], init[h], lab[h], l_ref)
        if nbad == 0:
            np.testing.assert_array_equal(cnt[h], n_ref)
            np.testing.assert_allclose(cent[h], c_ref, rtol=0, atol=1e-5 * np.abs(c_ref).max())


@pytest.mark.parametrize("cfg", ["tiny", "mid"])
def test_kmeans_all_iterations(layers, cfg):
    L = layers[cfg]
    w = L.workload
    cent, lab, cnt = ear.ear_kmeans(pu.dev(L.k, _tdt(w)), pu.dev(L.k_init), w.iters)
    cent, lab, cnt = pu.host(cent), pu.host(lab), pu.host(cnt)
    for h in range(L.k.shape[0]):
        c_ref, l_ref, n_ref = eo.kmeans(L.k[h], L.k_init[h], w.iters)
        c_prev, _, _ = eo.kmeans(L.k[h], L.k_init[h], w.iters - 1)
        bad = np.nonzero(lab[h] != l_ref)[0]
        # fp32 centroid sums drift ~1e-7 from the fp64 means; a differing final
        # label must be a near-tie under the oracle's previous centroids
        for i in bad:
            x = L.k[h][i].astype(np.float64)
            dg = ((x - c_prev[lab[h][i]]) ** 2).sum()
            dr = ((x - c_prev[l_ref[i]]) ** 2).sum()
            assert abs(dg - dr) <= 1e-4 * ((x ** 2).sum() + (c_prev[l_ref[i]] ** 2).sum())
        assert len(bad) <= 1e-3 * L.k.shape[1]
        assert cnt[h].sum() == L.k.shape[1]
        if len(bad) == 0:
            np.testing.assert_array_equal(cnt[h], n_ref)
            np.testing.assert_allclose(cent[h], c_ref, rtol=0, atol=1e-5 * np.abs(c_ref).max())


@pytest.mark.parametrize("n,c,d,iters", [(3001, 500, 64, 4), (2000, 300, 128, 3),
                                         (777, 17, 128, 5), (4096, 512, 128, 2),
                                         (5000, 700, 128, 2), (6000, 1000, 128, 2),
                                         (3000, 1500, 64, 2), (4096, 2048, 128, 1)])
def test_kmeans_tensor_core_path_shapes(n, c, d, iters):
    """bf16 k-means with C <= 2048 runs on the tensor cores: two 256-column
    chunks, a partial last column group, ragged row tiles, and beyond 512
    centroids passes of 512 with the row state carried between them (the
    pages' K_C = 1000 among them)."""
    w = gen.MID.with_(heads=2, n=n, d=d, n_centres=max(c // 3, 4), c_q=c, c_k=c, iters=iters)
    L = gen.make_layer(w)
    for it in (1, iters):
        cent, lab, cnt = ear.ear_kmeans(pu.dev(L.k, torch.bfloat16), pu.dev(L.k_init), it)
        cent, lab, cnt = pu.host(cent), pu.host(lab), pu.host(cnt)
        for h in range(2):
            c_ref, l_ref, n_ref = eo.kmeans(L.k[h], L.k_init[h], it)
            prev = L.k_init[h] if it == 1 else eo.kmeans(L.k[h], L.k_init[h], it - 1)[0]
            bad = np.nonzero(lab[h] != l_ref)[0]
            for i in bad:  # only near-ties under the centroids the last assignment used
                x = L.k[h][i].astype(np.float64)
                dg = ((x - prev[lab[h][i]]) ** 2).sum()
                dr = ((x - prev[l_ref[i]]) ** 2).sum()
                tol = pu.TIE_REL if it == 1 else 1e-4
                assert abs(dg - dr) <= tol * ((x ** 2).sum() + (prev[l_ref[i]] ** 2).sum())
            assert cnt[h].sum() == n
            np.testing.assert_array_equal(cnt[h], np.bincount(lab[h], minlength=c))
            if len(bad) == 0:
                np.testing.assert_allclose(cent[h], c_ref, rtol=0, atol=1e-5 * np.abs(c_ref).max())


def test_kmeans_rows_outside_fp16_are_decided_exactly():
    """Values with no exact fp16 copy (above 65504, or too small) send their
    rows through the fp64 decision; labels still match the oracle."""
    rng = np.random.default_rng(3)
    n, c, d = 1500, 40, 128
    x = rng.standard_normal((1, n, d))
    x[0, 10, 5] = 1.0e5
    x[0, 11, :] = 3.0e-8
    x[0, 12, 7] = -7.0e4
    x = gen.round_to_bf16(x)
    init = np.ascontiguousarray(x[:, rng.choice(n, c, replace=False)])
    init[0, 0] = x[0, 10]
    _, lab, _ = ear.ear_kmeans(pu.dev(x, torch.bfloat16), pu.dev(init), 1)
    _, l_ref, _ = eo.kmeans(x[0], init[0], 1)
    pu.assert_labels_exact_or_tie(x[0], init[0], pu.host(lab)[0], l_ref)


# --------------------------------------------------------------------------- permutation
@pytest.mark.parametrize("n,c,dtype,d", [(8192, 128, "bf16", 128), (1000, 7, "f32", 64),
                                         (3001, 40, "bf16", 64), (5, 3, "f32", 128)])
def test_permute_matches_oracle(n, c, dtype, d):
    rng = np.random.default_rng(n + c)
    bh = 3
    labels = rng.integers(0, c, (bh, n)).astype(np.int32)
    labels[labels == c // 2] = 0  # one empty cluster per slice
    x = gen.round_to_dtype(rng.standard_normal((bh, n, d)), dtype)
    perm, off, xp, mean = ear.ear_permute(pu.dev(labels), c, pu.dev(x, pu.torch_dtype(dtype)),
                                          seg_mean=True)
    perm, off, xp, mean = pu.host(perm), pu.host(off), pu.host(xp), pu.host(mean)
    for h in range(bh):
        p_ref, o_ref = eo.permute(labels[h], c)
        np.testing.assert_array_equal(perm[h], p_ref)
        np.testing.assert_array_equal(off[h], o_ref)
        np.testing.assert_array_equal(xp[h], x[h][p_ref])
        m_ref = eo.segment_mean(x[h], labels[h], c)
        np.testing.assert_allclose(mean[h], m_ref, rtol=0, atol=1e-6 * max(np.abs(m_ref).max(), 1))


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_permute_apply_reuses_a_permutation(dtype, d):
    """V laid out with K's permutation (no recount) equals the oracle's gather
    and segment means."""
    rng = np.random.default_rng(11)
    bh, n, c = 2, 3001, 41
    labels = rng.integers(0, c, (bh, n)).astype(np.int32)
    labels[labels == 5] = 6  # an empty cluster
    v = gen.round_to_dtype(rng.standard_normal((bh, n, d)), dtype)
    perm, off, _, _ = ear.ear_permute(pu.dev(labels), c)
    vp, mean = ear.ear_permute_apply(perm, off, pu.dev(v, pu.torch_dtype(dtype)), seg_mean=True)
    vp, mean = pu.host(vp), pu.host(mean)
    for h in range(bh):
        p_ref, _ = eo.permute(labels[h], c)
        np.testing.assert_array_equal(vp[h], v[h][p_ref])
        m_ref = eo.segment_mean(v[h], labels[h], c)
        np.testing.assert_allclose(mean[h], m_ref, rtol=0, atol=1e-6 * max(np.abs(m_ref).max(), 1))


def test_permute_bad_label_latches_device_status():
    labels = np.zeros((1, 100), np.int32)
    labels[0, 17] = 9  # out of range for C = 4
    perm, off, _, _ = ear.ear_permute(pu.dev(labels), 4)
    assert ear.ear_get_device_status() == 6  # EAR_ERR_DEVICE
    assert ear.ear_get_device_status() == 0  # cleared by the read
    assert pu.host(off)[0, -1] == 99


# --------------------------------------------------------------------------- probe
def _stack(runs, attr, dtype=None):
    a = np.stack([getattr(r, attr) for r in runs])
    return a.astype(dtype) if dtype is not None else a


@pytest.mark.parametrize("cfg", ["tiny", "mid"])
def test_probe_matches_oracle(layers, oracle_runs, cfg):
    L, runs = layers[cfg], oracle_runs[cfg]
    w = L.workload
    s = pu.scale_of(w.d)
    qc = _stack(runs, "q_cent", np.float32)
    kc = _stack(runs, "k_cent", np.float32)
    kx = np.stack([L.k[h][runs[h].k_perm] for h in range(len(runs))])
    e = ear.ear_probe(pu.dev(qc), pu.dev(_stack(runs, "q_counts", np.int32)), pu.dev(kc),
                      pu.dev(kx, _tdt(w)), pu.dev(_stack(runs, "k_offsets", np.int32)), s)
    e = pu.host(e)
    for h, r in enumerate(runs):
        e_ref = eo.probe(qc[h], r.q_counts, L.k[h], r.k_labels, kc[h], r.k_counts, s)
        np.testing.assert_allclose(e[h], e_ref, rtol=2e-5, atol=1e-7 * e_ref.max())


# --------------------------------------------------------------------------- route
def _route_case(e, qn, kn, nq, nk, density, mode):
    exact, bo, bl, pairs = ear.ear_route(pu.dev(e), pu.dev(qn), pu.dev(kn), nq, nk, density, mode)
    exact, bo, bl, pairs = pu.host(exact), pu.host(bo), pu.host(bl), pu.host(pairs)
    for h in range(e.shape[0]):
        ex_ref, p_ref = eo.route(e[h].astype(np.float64), qn[h], kn[h], nq, nk, density, mode)
        np.testing.assert_array_equal(exact[h], ex_ref)
        assert pairs[h] == p_ref
        o_ref, l_ref = eo.block_lists(ex_ref)
        np.testing.assert_array_equal(bo[h], o_ref)
        np.testing.assert_array_equal(bl[h][:o_ref[-1]], l_ref)


@pytest.mark.parametrize("cfg", ["tiny", "mid"])
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("density", [0.0, 0.05, 0.15, 0.25, 0.6, 1.0])
def test_route_given_same_error_is_bit_exact(oracle_runs, layers, cfg, mode, density):
    runs = oracle_runs[cfg]
    L = layers[cfg]
    e = _stack(runs, "e", np.float32)
    _route_case(e, _stack(runs, "q_counts", np.int32), _stack(runs, "k_counts", np.int32),
                L.q.shape[1], L.k.shape[1], density, mode)


# (37, 300), (100, 500): one 8-CTA cluster per slice with the keys in shared
# memory; (1100, 5) and (300, 500): too many query clusters / blocks for it, one
# block per slice with the keys in the workspace
@pytest.mark.parametrize("cq,ck", [(37, 300), (100, 500), (1100, 5), (300, 500)])
@pytest.mark.parametrize("seed", range(3))
@pytest.mark.parametrize("density", [0.0, 0.01, 0.3, 0.97, 1.0])
def test_route_ties_and_empty_clusters(seed, density, cq, ck):
    rng = np.random.default_rng(seed)
    bh = 4
    qn = rng.integers(0, 50, (bh, cq)).astype(np.int32)
    kn = rng.integers(0, 30, (bh, ck)).astype(np.int32)
    qn[:, 3] = 0
    kn[:, min(7, ck - 1)] = 0
    # few distinct values -> many exact ratio ties, broken by block index
    e = rng.integers(0, 5, (bh, cq, ck)).astype(np.float32) * np.float32(0.25)
    if ck > 12:
        e[:, :, 11] = e[:, :, 12]
    e = e * kn[:, None, :]  # equal E/|b| across many blocks in mode 0
    e *= (qn[:, :, None] > 0) * (kn[:, None, :] > 0)
    nq, nk = int(qn.sum(1).max()), int(kn.sum(1).max())
    for mode in (0, 1):
        _route_case(e.astype(np.float32), qn, kn, nq, nk, density, mode)


# --------------------------------------------------------------------------- attention
def _attention_inputs(L, runs):
    q = np.stack([L.q[h][r.q_perm] for h, r in enumerate(runs)])
    k = np.stack([L.k[h][r.k_perm] for h, r in enumerate(runs)])
    v = np.stack([L.v[h][r.k_perm] for h, r in enumerate(runs)])
    return q, k, v


def _run_attention(L, runs, compensate, exact=None, lists=None):
    w = L.workload
    t = _tdt(w)
    q, k, v = _attention_inputs(L, runs)
    ex = _stack(runs, "exact") if exact is None else exact
    if lists is None:
        bo = _stack(runs, "blk_offsets", np.int32)
        bl = np.stack([np.pad(r.blk_list, (0, ex.shape[1] * ex.shape[2] - len(r.blk_list)))
                       for r in runs]).astype(np.int32)
    else:
        bo, bl = lists
    o, lse = ear.ear_attention(
        pu.dev(q, t), pu.dev(k, t), pu.dev(v, t), pu.dev(_stack(runs, "q_offsets", np.int32)),
        pu.dev(_stack(runs, "k_offsets", np.int32)), pu.dev(_stack(runs, "q_perm", np.int32)),
        pu.dev(_stack(runs, "k_cent", np.float32)), pu.dev(_stack(runs, "v_mean", np.float32)),
        pu.dev(np.ascontiguousarray(ex)), pu.dev(bo), pu.dev(bl), pu.scale_of(w.d), compensate,
        want_lse=True)
    return pu.host(o), pu.host(lse)


@pytest.mark.parametrize("cfg", ["tiny", "mid"])
@pytest.mark.parametrize("compensate", [True, False])
def test_attention_given_same_mask(layers, oracle_runs, cfg, compensate):
    L, runs = layers[cfg], oracle_runs[cfg]
    w = L.workload
    o, lse = _run_attention(L, runs, compensate)
    for h, r in enumerate(runs):
        o_ref, lse_ref = eo.attention(L.q[h], L.k[h], L.v[h], r.q_labels, r.k_labels, r.k_cent,
                                      r.v_mean, r.k_counts, r.exact, pu.scale_of(w.d), compensate)
        ok = np.isfinite(lse_ref)
        pu.assert_attention_close(o[h][ok], o_ref[ok], w.dtype)
        assert np.all(o[h][~ok] == 0) and np.all(np.isneginf(lse[h][~ok]))
        np.testing.assert_allclose(lse[h][ok], lse_ref[ok], rtol=0, atol=pu.LSE_TOL[w.dtype])


@pytest.mark.parametrize("compensate", [True, False])
@pytest.mark.parametrize("ck,density", [(400, 0.3), (37, 0.5), (250, 0.05)])
def test_attention_packs_small_key_clusters(compensate, ck, density):
    """Many small key clusters: most 32-row boxes are partial and one chunk
    gathers boxes of several clusters (bf16 tensor-core path)."""
    w = gen.MID.with_(heads=2, n=2000, d=128, n_centres=60, c_q=7, c_k=ck, iters=2,
                      density=density)
    L = gen.make_layer(w)
    runs = [eo.pipeline(L.q[h], L.k[h], L.v[h], L.q_init[h], L.k_init[h], w.iters, w.density,
                        compensate=compensate) for h in range(2)]
    o, lse = _run_attention(L, runs, compensate)
    for h, r in enumerate(runs):
        ok = np.isfinite(r.lse)
        pu.assert_attention_close(o[h][ok], r.o[ok], "bf16")
        np.testing.assert_allclose(lse[h][ok], r.lse[ok], rtol=0, atol=pu.LSE_TOL["bf16"])


# --------------------------------------------------------------------------- whole layer
@pytest.mark.parametrize("cfg", ["tiny", "mid"])
def test_layer_end_to_end(layers, oracle_runs, cfg):
    L, runs = layers[cfg], oracle_runs[cfg]
    w = L.workload
    t = _tdt(w)
    res = ear.ear_layer(pu.dev(L.q, t), pu.dev(L.k, t), pu.dev(L.v, t), pu.dev(L.q_init),
                        pu.dev(L.k_init), w.iters, w.density, want_lse=True)
    o = pu.host(res.o)
    qlab, klab = pu.host(res.q_labels), pu.host(res.k_labels)
    exact, e = pu.host(res.exact), pu.host(res.e)
    pairs = pu.host(res.exact_pairs)
    budget = math.floor(w.density * float(L.q.shape[1] * L.k.shape[1]))
    for h, r in enumerate(runs):
        assert pairs[h] <= budget
        assert (qlab[h] != r.q_labels).mean() <= 1e-3 and (klab[h] != r.k_labels).mean() <= 1e-3
        # blocks may differ only at ratio ties (the centroids carry fp32 rounding)
        diff = np.argwhere(exact[h] != r.exact)
        if len(diff):
            rr = pu.route_ratio(r.e, r.q_counts, r.k_counts, 0)
            cut = rr[r.exact.astype(bool)].min()
            for a, b in diff:
                assert abs(rr[a, b] - cut) <= 1e-4 * cut
        same_rows = (exact[h] == r.exact).all(axis=1)
        keep = (qlab[h] == r.q_labels) & same_rows[r.q_labels]
        assert keep.mean() > 0.9
        pu.assert_attention_close(o[h][keep], r.o[keep], w.dtype)
        # E against the oracle's probe with the GPU's own centroids and labels
        qc, kc = pu.host(res.q_centroids)[h], pu.host(res.k_centroids)[h]
        e_ref = eo.probe(qc, pu.host(res.q_counts)[h], L.k[h], klab[h], kc,
                         pu.host(res.k_counts)[h], pu.scale_of(w.d))
        np.testing.assert_allclose(e[h], e_ref, rtol=2e-5, atol=1e-7 * e_ref.max())


# --------------------------------------------------------------------------- edge cases
def _dense(q, k, v, s):
    z = s * q.astype(np.float64) @ k.astype(np.float64).T
    z -= z.max(1, keepdims=True)
    p = np.exp(z)
    return (p / p.sum(1, keepdims=True)) @ v.astype(np.float64)


@pytest.mark.parametrize("dtype,d", [("f32", 64), ("bf16", 128), ("bf16", 64), ("f32", 128)])
def test_full_density_ragged_unequal_lengths_is_dense(dtype, d):
    rng = np.random.default_rng(5)
    nq, nk, cq, ck = 701, 1000, 9, 23
    q = gen.round_to_dtype(rng.standard_normal((2, nq, d)), dtype)
    k = gen.round_to_dtype(rng.standard_normal((2, nk, d)), dtype)
    v = gen.round_to_dtype(rng.standard_normal((2, nk, d)), dtype)
    qi = np.ascontiguousarray(q[:, :cq])
    ki = np.ascontiguousarray(k[:, :ck])
    t = pu.torch_dtype(dtype)
    res = ear.ear_layer(pu.dev(q, t), pu.dev(k, t), pu.dev(v, t), pu.dev(qi), pu.dev(ki), 3, 1.0)
    assert (pu.host(res.exact_pairs) == nq * nk).all()
    o = pu.host(res.o)
    for h in range(2):
        pu.assert_attention_close(o[h], _dense(q[h], k[h], v[h], 1 / math.sqrt(d)), dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_zero_density_one_key_cluster_is_mean_value(dtype):
    rng = np.random.default_rng(6)
    q = gen.round_to_dtype(rng.standard_normal((1, 300, 128)), dtype)
    k = gen.round_to_dtype(rng.standard_normal((1, 257, 128)), dtype)
    v = gen.round_to_dtype(rng.standard_normal((1, 257, 128)), dtype)
    t = pu.torch_dtype(dtype)
    res = ear.ear_layer(pu.dev(q, t), pu.dev(k, t), pu.dev(v, t), pu.dev(q[:, :4].copy()),
                        pu.dev(k[:, :1].copy()), 2, 0.0)
    assert pu.host(res.exact).sum() == 0
    mean = v[0].astype(np.float64).mean(0)
    tol = 1e-4 if dtype == "f32" else 1e-2
    np.testing.assert_allclose(pu.host(res.o)[0], np.broadcast_to(mean, (300, 128)), atol=tol)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("density", [0.0, 0.2])
def test_singleton_key_clusters_and_empty_clusters(dtype, density):
    """C_k = N_k with init = the keys (compensation exact) plus duplicated init
    rows on the query side (clusters that stay empty)."""
    rng = np.random.default_rng(8)
    nq, nk, d = 200, 256, 64
    q = gen.round_to_dtype(rng.standard_normal((1, nq, d)), dtype)
    k = gen.round_to_dtype(rng.standard_normal((1, nk, d)), dtype)
    v = gen.round_to_dtype(rng.standard_normal((1, nk, d)), dtype)
    qi = np.concatenate([q[:, :5], q[:, :5]], axis=1)  # clusters 5..9 duplicate 0..4: empty
    t = pu.torch_dtype(dtype)
    res = ear.ear_layer(pu.dev(q, t), pu.dev(k, t), pu.dev(v, t), pu.dev(qi), pu.dev(k.copy()), 1,
                        density)
    qn = pu.host(res.q_counts)[0]
    assert (qn[5:] == 0).all() and (pu.host(res.k_counts) == 1).all()
    pu.assert_attention_close(pu.host(res.o)[0], _dense(q[0], k[0], v[0], 1 / math.sqrt(d)), dtype)


# --------------------------------------------------------------------------- full size, sampled
@pytest.mark.slow
def test_wan_layer_full_size_sampled():
    """The 40-head Wan2.x layer (N = 75,600, C_q = 100, C_k = 500, rho = 0.10) in
    the launch configuration the benchmark times; sampled checks per step."""
    w = gen.WAN
    L = gen.make_layer(w)
    t = torch.bfloat16
    q, k, v = pu.dev(L.q, t), pu.dev(L.k, t), pu.dev(L.v, t)
    res = ear.ear_layer(q, k, v, pu.dev(L.q_init), pu.dev(L.k_init), w.iters, w.density,
                        want_lse=True)
    torch.cuda.synchronize()
    assert ear.ear_get_device_status() == 0
    s = pu.scale_of(w.d)
    one = ear.ear_kmeans(k, pu.dev(L.k_init), 1)[1]
    one = pu.host(one)
    o = pu.host(res.o)
    rng = np.random.default_rng(0)
    for h in (0, w.heads - 1):
        # k-means iteration 1 on sampled rows: assignment from the seeded init
        rows = rng.choice(w.n, 2000, replace=False)
        _, l_ref, _ = eo.kmeans(L.k[h][rows], L.k_init[h], 1)
        pu.assert_labels_exact_or_tie(L.k[h][rows], L.k_init[h], one[h][rows], l_ref)
        # permutation: stable and consistent with the labels
        qlab, qperm = pu.host(res.q_labels)[h], pu.host(res.q_perm)[h]
        p_ref, o_ref = eo.permute(qlab, w.c_q)
        np.testing.assert_array_equal(qperm, p_ref)
        np.testing.assert_array_equal(pu.host(res.q_offsets)[h], o_ref)
        # probe with the GPU's centroids, route given the GPU's E
        qn, kn = pu.host(res.q_counts)[h], pu.host(res.k_counts)[h]
        klab = pu.host(res.k_labels)[h]
        qc, kc = pu.host(res.q_centroids)[h], pu.host(res.k_centroids)[h]
        e = pu.host(res.e)[h]
        e_ref = eo.probe(qc, qn, L.k[h], klab, kc, kn, s)
        np.testing.assert_allclose(e, e_ref, rtol=2e-5, atol=1e-7 * e_ref.max())
        ex_ref, pairs_ref = eo.route(e.astype(np.float64), qn, kn, w.n, w.n, w.density)
        np.testing.assert_array_equal(pu.host(res.exact)[h], ex_ref)
        assert pu.host(res.exact_pairs)[h] == pairs_ref
        # attention on sampled queries given the GPU's mask, labels and centroids
        qi = rng.choice(w.n, 384, replace=False)
        vm = eo.segment_mean(L.v[h], klab, w.c_k)
        o_ref, _ = eo.attention(L.q[h][qi], L.k[h], L.v[h], qlab[qi], klab, kc, vm, kn, ex_ref, s)
        pu.assert_attention_close(o[h][qi], o_ref, "bf16")


# --------------------------------------------------------------------------- probe -> route
def _probe_route_case(q, k, qi, ki, iters, d, densities, dtype):
    """Oracle k-means and permutation; then ear_probe and ear_route on the GPU
    from the oracle's centroids (rounded to fp32, the ABI's type), counts and
    permuted keys, against eo.route(eo.probe(...)) on the same values.  A
    routed block may differ only at a ratio tie within 1e-6 of the oracle's
    cut; the lists, offsets and pair count must describe the GPU's own mask."""
    bh = len(q)
    s = pu.scale_of(d)
    runs = []
    for h in range(bh):
        qc, ql, qn = eo.kmeans(q[h], qi[h], iters)
        kc, kl, kn = eo.kmeans(k[h], ki[h], iters)
        kp, ko = eo.permute(kl, ki.shape[1])
        runs.append((qc.astype(np.float32), qn.astype(np.int32), kc.astype(np.float32), kl,
                     kn.astype(np.int32), kp, ko.astype(np.int32)))
    t = pu.torch_dtype(dtype)
    qc = np.stack([r[0] for r in runs])
    qn = np.stack([r[1] for r in runs])
    kc = np.stack([r[2] for r in runs])
    kn = np.stack([r[4] for r in runs])
    kx = np.stack([k[h][runs[h][5]] for h in range(bh)])
    ko = np.stack([r[6] for r in runs])
    e = ear.ear_probe(pu.dev(qc), pu.dev(qn), pu.dev(kc), pu.dev(kx, t), pu.dev(ko), s)
    e_ref = [eo.probe(qc[h], qn[h], k[h], runs[h][3], kc[h], kn[h], s) for h in range(bh)]
    nq, nk = q.shape[1], k.shape[1]
    ndiff = 0
    for mode in (0, 1):
        for rho in densities:
            exact, bo, bl, pairs = ear.ear_route(e, pu.dev(qn), pu.dev(kn), nq, nk, rho, mode)
            exact, bo, bl, pairs = pu.host(exact), pu.host(bo), pu.host(bl), pu.host(pairs)
            for h in range(bh):
                ex_ref, p_ref = eo.route(e_ref[h], qn[h], kn[h], nq, nk, rho, mode)
                nd = pu.assert_route_exact_or_tie(exact[h], ex_ref, e_ref[h], qn[h], kn[h], mode)
                ndiff += nd
                if nd == 0:
                    assert pairs[h] == p_ref
                o_own, l_own = eo.block_lists(exact[h])
                np.testing.assert_array_equal(bo[h], o_own)
                np.testing.assert_array_equal(bl[h][:o_own[-1]], l_own)
                cost = (qn[h][:, None].astype(np.int64) * kn[h][None, :])[exact[h].astype(bool)]
                assert pairs[h] == cost.sum() <= math.floor(rho * float(nq * nk))
    return ndiff


@pytest.mark.parametrize("cfg", ["tiny", "mid"])
def test_probe_then_route_given_oracle_clustering(layers, cfg):
    L = layers[cfg]
    w = L.workload
    _probe_route_case(L.q, L.k, L.q_init, L.k_init, w.iters, w.d,
                      (0.0, 0.02, 0.05, 0.1, 0.15, 0.25, 0.5, 0.9, 1.0), w.dtype)


@pytest.mark.slow
def test_wan_probe_then_route_given_oracle_clustering():
    """Two Wan2.x heads (N = 75,600, C_q = 100, C_k = 500): the GPU probe and
    route from the oracle's clustering reproduce the oracle's routed blocks."""
    w = gen.WAN
    L = gen.make_layer(w, heads=[0, w.heads - 1])
    _probe_route_case(L.q, L.k, L.q_init, L.k_init, w.iters, w.d, (0.05, 0.1, 0.2, 0.4), w.dtype)


# --------------------------------------------------------------------------- attention paths
def _direct_attention(q, k, v, q_sizes, k_sizes, exact, compensate, seed_dtype="bf16"):
    """Runs ear_attention on hand-built clusters (tokens already grouped by
    cluster, q_perm = identity) and returns (o, lse, oracle o, oracle lse)."""
    d = q.shape[1]
    t = pu.torch_dtype(seed_dtype)
    qo = np.concatenate([[0], np.cumsum(q_sizes)]).astype(np.int32)
    ko = np.concatenate([[0], np.cumsum(k_sizes)]).astype(np.int32)
    ql = np.repeat(np.arange(len(q_sizes)), q_sizes).astype(np.int32)
    kl = np.repeat(np.arange(len(k_sizes)), k_sizes).astype(np.int32)
    kc = eo.segment_mean(k, kl, len(k_sizes)).astype(np.float32)
    vm = eo.segment_mean(v, kl, len(k_sizes)).astype(np.float32)
    o_lists, l_lists = eo.block_lists(exact)
    bl = np.zeros(exact.size, np.int32)
    bl[:len(l_lists)] = l_lists
    s = pu.scale_of(d)
    o, lse = ear.ear_attention(
        pu.dev(q[None], t), pu.dev(k[None], t), pu.dev(v[None], t), pu.dev(qo[None]),
        pu.dev(ko[None]), pu.dev(np.arange(len(q), dtype=np.int32)[None]), pu.dev(kc[None]),
        pu.dev(vm[None]), pu.dev(exact[None].astype(np.uint8)), pu.dev(o_lists[None].astype(np.int32)),
        pu.dev(bl[None]), s, compensate, want_lse=True)
    o_ref, lse_ref = eo.attention(q, k, v, ql, kl, kc, vm, np.asarray(k_sizes, np.int64),
                                  exact.astype(np.uint8), s, compensate)
    return pu.host(o)[0], pu.host(lse)[0], o_ref, lse_ref


@pytest.mark.parametrize("pattern", ["all_exact", "mixed"])
def test_attention_running_max_rescale_path(pattern):
    """Every later key cluster raises the logits by about 9.8 in base 2, more
    than the kernel's 2^8 rescale threshold, so the running max moves and O is
    rescaled in tensor memory on almost every chunk (and on centroid chunks in
    the mixed case)."""
    rng = np.random.default_rng(77)
    d = 128
    q_sizes = [300]
    k_sizes = [40, 64, 70, 33, 64, 50]
    q = gen.round_to_bf16(0.5 * rng.standard_normal((300, d)) + 1.0)
    shift = np.repeat(0.6 * np.arange(len(k_sizes)), k_sizes)[:, None]
    k = gen.round_to_bf16(0.5 * rng.standard_normal((sum(k_sizes), d)) + shift)
    v = gen.round_to_bf16(rng.standard_normal((sum(k_sizes), d)))
    exact = np.ones((1, len(k_sizes)), np.uint8)
    if pattern == "mixed":
        exact[0, [2, 4]] = 0
    o, lse, o_ref, lse_ref = _direct_attention(q, k, v, q_sizes, k_sizes, exact, True)
    pu.assert_attention_close(o, o_ref, "bf16")
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=pu.LSE_TOL["bf16"])


@pytest.mark.parametrize("compensate", [True, False])
def test_attention_block_lists_beyond_shared_memory(compensate):
    """C_k = 2,100 key clusters of 1-3 keys: the unit's block list and the
    slice's key offsets exceed the 2,048 entries staged in shared memory, so
    the kernel walks them in global memory."""
    rng = np.random.default_rng(91)
    d = 64
    q_sizes = [130, 70]
    k_sizes = rng.integers(1, 4, 2100)
    q = gen.round_to_bf16(rng.standard_normal((sum(q_sizes), d)))
    k = gen.round_to_bf16(rng.standard_normal((int(k_sizes.sum()), d)))
    v = gen.round_to_bf16(rng.standard_normal((int(k_sizes.sum()), d)))
    exact = np.zeros((2, len(k_sizes)), np.uint8)
    exact[0] = 1                                   # 2,100 listed clusters
    exact[1] = rng.integers(0, 2, len(k_sizes))    # about half
    o, lse, o_ref, lse_ref = _direct_attention(q, k, v, q_sizes, k_sizes, exact, compensate)
    pu.assert_attention_close(o, o_ref, "bf16")
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=pu.LSE_TOL["bf16"])


def test_compensated_logits_keep_fp32_centroids(layers, oracle_runs):
    """At density 0 every term is compensated, so lse = log sum_b |b| e^{s q·k̄_b}
    isolates the centroid logits: with k̄ as a bf16 hi + lo pair they stay
    within 1e-4 of the oracle's fp64 values (one bf16 copy would be ~2e-3 off)."""
    L, runs = layers["mid"], oracle_runs["mid"]
    w = L.workload
    none = np.zeros_like(_stack(runs, "exact"))
    lists = (np.zeros((len(runs), w.c_q + 1), np.int32), np.zeros((len(runs), w.c_q * w.c_k), np.int32))
    o, lse = _run_attention(L, runs, True, exact=none, lists=lists)
    worst = 0.0
    for h, r in enumerate(runs):
        o_ref, lse_ref = eo.attention(L.q[h], L.k[h], L.v[h], r.q_labels, r.k_labels,
                                      r.k_cent.astype(np.float32), r.v_mean.astype(np.float32),
                                      r.k_counts, none[h], pu.scale_of(w.d), True)
        worst = max(worst, float(np.abs(lse[h] - lse_ref).max()))
        pu.assert_attention_close(o[h], o_ref, "bf16")
    print(f"compensated lse max-abs error vs fp64: {worst:.3e}")
    assert worst <= 1e-4


# --------------------------------------------------------------------------- weight probes
@pytest.mark.parametrize("mode", [1, 2])
def test_weight_probes_match_oracle(layers, oracle_runs, mode):
    """The unnormalized-weight and value-aware probes (SVG-EAR §4.2, §4.3) on
    the tensor cores, given the oracle's clustering (mid configuration, bf16).
    The GPU sums fp32 terms (expm1f of the logit gap, then the w̄^2 factor), so
    E is compared at rtol 1e-4 (about 10^2 fp32 roundings per block); blocks
    far below the row's largest logit fall under fp32's range and are compared
    against 1e-7 of the largest E."""
    L, runs = layers["mid"], oracle_runs["mid"]
    w = L.workload
    s = pu.scale_of(w.d)
    qc = _stack(runs, "q_cent", np.float32)
    kc = _stack(runs, "k_cent", np.float32)
    vm = _stack(runs, "v_mean", np.float32)
    kx = np.stack([L.k[h][r.k_perm] for h, r in enumerate(runs)])
    vx = np.stack([L.v[h][r.k_perm] for h, r in enumerate(runs)])
    e = ear.ear_probe(pu.dev(qc), pu.dev(_stack(runs, "q_counts", np.int32)), pu.dev(kc),
                      pu.dev(kx, torch.bfloat16), pu.dev(_stack(runs, "k_offsets", np.int32)), s,
                      mode=mode, v_perm=pu.dev(vx, torch.bfloat16), v_centroids=pu.dev(vm))
    e = pu.host(e)
    for h, r in enumerate(runs):
        e_ref = eo.probe_weights(qc[h], r.q_counts, L.k[h], r.k_labels, kc[h], r.k_counts,
                                 L.v[h], vm[h], s, mode)
        np.testing.assert_allclose(e[h], e_ref, rtol=1e-4, atol=1e-7 * e_ref.max())
        # routed on these estimates, the GPU and the oracle pick the same blocks
        # except at ratios within the comparison's 1e-4
        for rho in (0.05, 0.15, 0.3):
            ex, _, _, _ = ear.ear_route(pu.dev(e[h][None]), pu.dev(r.q_counts[None].astype(np.int32)),
                                        pu.dev(r.k_counts[None].astype(np.int32)), w.n, w.n, rho)
            ex_ref, _ = eo.route(e_ref, r.q_counts, r.k_counts, w.n, w.n, rho)
            diff = np.argwhere(pu.host(ex)[0] != ex_ref)
            if len(diff):
                rr = pu.route_ratio(e_ref, r.q_counts, r.k_counts, 0)
                cut = rr[ex_ref.astype(bool)].min()
                for a, b in diff:
                    assert abs(rr[a, b] - cut) <= 1e-4 * cut


@pytest.mark.parametrize("mode", [1, 2])
def test_weight_probes_vanish_on_constant_clusters(mode):
    """P2 on the GPU: keys and values equal to their cluster means give E = 0 up
    to the fp32 logit gap (|g| <~ 1e-4 at d = 128 here), i.e. E <= |b| g^2 (1 + |v̄|^2)
    ~ 5e-5; a non-constant block is O(1) or larger."""
    rng = np.random.default_rng(21)
    d, ck, per, cq = 128, 7, 40, 5
    kc = gen.round_to_bf16(rng.standard_normal((ck, d)))
    vc = gen.round_to_bf16(rng.standard_normal((ck, d)))
    k = np.repeat(kc, per, axis=0)[None]
    v = np.repeat(vc, per, axis=0)[None]
    ko = (np.arange(ck + 1) * per).astype(np.int32)[None]
    qc = rng.standard_normal((1, cq, d)).astype(np.float32)
    qn = np.full((1, cq), 3, np.int32)
    e = ear.ear_probe(pu.dev(qc), pu.dev(qn), pu.dev(kc[None]), pu.dev(k, torch.bfloat16),
                      pu.dev(ko), 0.2, mode=mode, v_perm=pu.dev(v, torch.bfloat16),
                      v_centroids=pu.dev(vc[None]))
    assert np.abs(pu.host(e)).max() <= 1e-4


# --------------------------------------------------------------------------- per-query-cluster budgets
@pytest.mark.parametrize("cfg", ["tiny", "mid"])
@pytest.mark.parametrize("rho", [0.0, 0.05, 0.15, 0.4, 1.0])
def test_route_rows_given_same_error_is_bit_exact(oracle_runs, layers, cfg, rho):
    """Per-query-cluster routing (SVG-EAR §5 "Implementation") under each query
    cluster's share of the budget: given the oracle's E, the GPU's exact mask,
    lists and pair count are the oracle's."""
    runs = oracle_runs[cfg]
    L = layers[cfg]
    nk = L.k.shape[1]
    e = _stack(runs, "e", np.float32)
    qn = _stack(runs, "q_counts", np.int32)
    kn = _stack(runs, "k_counts", np.int32)
    budget = ear.ear_uniform_budget(pu.dev(qn), nk, rho)
    b_ref = np.stack([eo.uniform_row_budget(qn[h], nk, rho) for h in range(len(runs))])
    np.testing.assert_array_equal(pu.host(budget), b_ref)
    exact, bo, bl, pairs = ear.ear_route_rows(pu.dev(e), pu.dev(qn), pu.dev(kn), budget)
    exact, bo, bl, pairs = pu.host(exact), pu.host(bo), pu.host(bl), pu.host(pairs)
    for h in range(len(runs)):
        ex_ref, p_ref = eo.route_rows(e[h].astype(np.float64), qn[h], kn[h], b_ref[h])
        np.testing.assert_array_equal(exact[h], ex_ref)
        assert pairs[h] == p_ref.sum()
        o_ref, l_ref = eo.block_lists(ex_ref)
        np.testing.assert_array_equal(bo[h], o_ref)
        np.testing.assert_array_equal(bl[h][:o_ref[-1]], l_ref)


@pytest.mark.parametrize("seed", range(2))
def test_route_rows_ties_empty_clusters_and_budgets(seed):
    rng = np.random.default_rng(100 + seed)
    bh, cq, ck = 3, 37, 300
    qn = rng.integers(0, 40, (bh, cq)).astype(np.int32)
    kn = rng.integers(0, 25, (bh, ck)).astype(np.int32)
    qn[:, 2] = 0
    kn[:, 5] = 0
    e = (rng.integers(0, 4, (bh, cq, ck)) * kn[:, None, :]).astype(np.float32)  # ratio ties
    budget = rng.integers(0, 20000, (bh, cq)).astype(np.int64)
    exact, bo, bl, pairs = ear.ear_route_rows(pu.dev(e), pu.dev(qn), pu.dev(kn), pu.dev(budget))
    exact, pairs = pu.host(exact), pu.host(pairs)
    for h in range(bh):
        ex_ref, p_ref = eo.route_rows(e[h].astype(np.float64), qn[h], kn[h], budget[h])
        np.testing.assert_array_equal(exact[h], ex_ref)
        assert pairs[h] == p_ref.sum()


@pytest.mark.parametrize("p", [0.3, 0.7, 0.85, 0.95, 1.0])
def test_topp_budget_matches_oracle(oracle_runs, p):
    """SVG2-style top-p budgets from the centroid attention mass (fp64 on both
    sides; a budget may differ only where the oracle's cumulative mass at the
    cut is within 1e-12 of p times the total)."""
    runs = oracle_runs["mid"]
    s = float(np.float32(pu.scale_of(128)))
    qc = _stack(runs, "q_cent", np.float32)
    kc = _stack(runs, "k_cent", np.float32)
    qn = _stack(runs, "q_counts", np.int32)
    kn = _stack(runs, "k_counts", np.int32)
    got = pu.host(ear.ear_topp_budget(pu.dev(qc), pu.dev(qn), pu.dev(kc), pu.dev(kn), p, s))
    for h in range(len(runs)):
        ref = eo.topp_budget(qc[h], qn[h], kc[h], kn[h], s, p)
        for a in np.nonzero(got[h] != ref)[0]:
            live = kn[h] > 0
            z = s * qc[h][a].astype(np.float64) @ kc[h][live].astype(np.float64).T
            w = kn[h][live] * np.exp(z - z.max())
            cum = np.cumsum(np.sort(w)[::-1])
            assert np.min(np.abs(cum - p * w.sum())) <= 1e-12 * w.sum()
    # top-p sets: E = mass x |b| routed under these budgets selects exactly them
    b = ear.ear_topp_budget(pu.dev(qc), pu.dev(qn), pu.dev(kc), pu.dev(kn), p, s)
    mass = np.zeros((len(runs), qc.shape[1], kc.shape[1]), np.float32)
    for h in range(len(runs)):
        z = s * qc[h].astype(np.float64) @ kc[h].astype(np.float64).T
        m = kn[h][None, :] * np.exp(z - z.max(axis=1, keepdims=True))
        mass[h] = (m * kn[h][None, :]).astype(np.float32)
    exact, _, _, pairs = ear.ear_route_rows(pu.dev(mass), pu.dev(qn), pu.dev(kn), b)
    assert (pu.host(pairs) == pu.host(b).sum(axis=1)).all()


# --------------------------------------------------------------------------- diagnostics
@pytest.mark.parametrize("cfg", ["tiny", "mid"])
def test_cluster_stats_match_oracle(layers, oracle_runs, cfg):
    """δ^2 and K_max (SVG-EAR §4.2 bound residual, §5.3) of the oracle's
    clustering: rows in fp32, sums in fp64, so rtol 1e-5."""
    L, runs = layers[cfg], oracle_runs[cfg]
    w = L.workload
    t = _tdt(w)
    for x, lab, cen in ((L.q, "q_labels", "q_cent"), (L.k, "k_labels", "k_cent")):
        labels = _stack(runs, lab, np.int32)
        cent = _stack(runs, cen, np.float32)
        ms, mx = ear.ear_cluster_stats(pu.dev(x, t), pu.dev(labels), pu.dev(cent))
        ms, mx = pu.host(ms), pu.host(mx)
        for h in range(len(runs)):
            ref_ms, ref_mx = eo.cluster_stats(x[h], labels[h], cent[h])
            np.testing.assert_allclose(ms[h], ref_ms, rtol=1e-5)
            np.testing.assert_allclose(mx[h], ref_mx, rtol=1e-6)
        r = ear.bound_residual(ms, mx, x.shape[1], w.d)
        np.testing.assert_allclose(r, [eo.bound_residual(a, b, x.shape[1], w.d)
                                       for a, b in zip(ms, mx)], rtol=1e-12)


def test_normalizer_change_matches_oracle(layers, oracle_runs):
    """The SVG-EAR §5.1 statistic from the library's own lse: the routed layer
    against every block exact (dense), compared with the oracle's formula."""
    L, runs = layers["mid"], oracle_runs["mid"]
    full = np.ones_like(_stack(runs, "exact"))
    lists = (np.stack([eo.block_lists(full[h])[0] for h in range(len(runs))]).astype(np.int32),
             np.stack([eo.block_lists(full[h])[1] for h in range(len(runs))]).astype(np.int32))
    _, lse_s = _run_attention(L, runs, True)
    _, lse_d = _run_attention(L, runs, True, exact=full, lists=lists)
    got = pu.host(ear.ear_normalizer_change(pu.dev(lse_s), pu.dev(lse_d)))
    for h in range(len(runs)):
        ref = eo.normalizer_change(lse_s[h], lse_d[h])
        np.testing.assert_allclose(got[h], ref, rtol=1e-9)
    assert np.all(got > 0) and np.all(got < 1)
