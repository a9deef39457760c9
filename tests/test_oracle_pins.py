"""Pins of the fp64 CPU oracle against things other than itself (CPU only).

Each test names the fact it checks: a closed form the pages fix, an invariant,
a special case that reduces to a textbook or library routine, a hand-worked
example (tests/golden/hand_worked.json), or the independent token-level brute
force in tests/bruteforce.py.  Citations "SVG-EAR §x" are to the paper
"SVG-EAR: Parameter-Free Linear Compensation for Sparse Video Generation via
Error-aware Routing", by section.
"""
import json
import math
import os
import warnings

import numpy as np
import pytest

import bruteforce as bf
from oracle import ear_oracle as eo

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _mixture(rng, n, d, centres, sigma):
    mu = rng.standard_normal((centres, d))
    z = rng.integers(0, centres, n)
    return mu[z] + sigma * rng.standard_normal((n, d))


def _head(seed, nq=48, nk=40, d=8, cq=4, ck=5, iters=4, centres=6):
    rng = np.random.default_rng(seed)
    q = _mixture(rng, nq, d, centres, 0.3)
    k = _mixture(rng, nk, d, centres, 0.3)
    v = rng.standard_normal((nk, d))
    qi = q[rng.choice(nq, cq, replace=False)]
    ki = k[rng.choice(nk, ck, replace=False)]
    return q, k, v, qi, ki, iters


# --------------------------------------------------------------------------- golden
def test_golden_kmeans_one_step():
    g = _golden()["kmeans_one_step"]
    c, l, n = eo.kmeans(np.array(g["x"], float), np.array(g["init"], float), g["iters"])
    assert l.tolist() == g["labels"]
    assert n.tolist() == g["counts"]
    np.testing.assert_array_equal(c, np.array(g["centroids"], float))


def test_golden_kmeans_tie_and_empty():
    g = _golden()["kmeans_tie_and_empty"]
    c, l, n = eo.kmeans(np.array(g["x"], float), np.array(g["init"], float), g["iters"])
    assert l.tolist() == g["labels"]
    assert n.tolist() == g["counts"]
    np.testing.assert_array_equal(c, np.array(g["centroids"], float))


def test_golden_permute():
    g = _golden()["permute"]
    p, o = eo.permute(np.array(g["labels"]), g["n_clusters"])
    assert p.tolist() == g["perm"]
    assert o.tolist() == g["offsets"]


def test_golden_two_by_two_pipeline_steps():
    g = _golden()["two_by_two"]
    s = 1 / math.sqrt(2)
    q, k, v = (np.array(g[x], float) for x in ("q", "k", "v"))
    ql, kl = np.array(g["q_labels"]), np.array(g["k_labels"])
    qc, kc = np.array(g["q_centroids"], float), np.array(g["k_centroids"], float)
    qn, kn = np.array([2]), np.array([2, 2])
    vm = eo.segment_mean(v, kl, 2)
    np.testing.assert_allclose(vm, np.array(g["v_means"], float), rtol=0, atol=1e-15)
    e = eo.probe(qc, qn, k, kl, kc, kn, s)
    np.testing.assert_allclose(e, np.array(g["E"]), rtol=1e-15, atol=1e-15)
    exact, pairs = eo.route(e, qn, kn, 2, 4, g["density"])
    assert exact.tolist() == g["exact"] and pairs == g["exact_pairs"]
    o, _ = eo.attention(q, k, v, ql, kl, kc, vm, kn, exact, s)
    es, e3, e2, em2 = math.exp(s), math.exp(3 * s), math.exp(2 * s), math.exp(-2 * s)
    o0 = (es * np.array([1, 0]) + e3 * np.array([0, 1]) + 2 * e2 * np.array([3, 1])) / (es + e3 + 2 * e2)
    o1 = (es * np.array([1, 0]) + e3 * np.array([0, 1]) + 2 * em2 * np.array([3, 1])) / (es + e3 + 2 * em2)
    np.testing.assert_allclose(o, np.stack([o0, o1]), rtol=1e-14, atol=1e-14)


# --------------------------------------------------------------------------- P1: rho = 1 is dense
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_p1_full_density_is_dense_attention(seed):
    q, k, v, qi, ki, it = _head(seed)
    r = eo.pipeline(q, k, v, qi, ki, it, density=1.0)
    assert r.exact_pairs == q.shape[0] * k.shape[0]
    ref = bf.dense_attention(q, k, v, 1 / math.sqrt(q.shape[1]))
    np.testing.assert_allclose(r.o, ref, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------- P2: duplicated clusters
@pytest.mark.parametrize("density", [0.0, 0.1, 0.37, 0.8])
def test_p2_constant_clusters_compensate_exactly(density):
    rng = np.random.default_rng(7)
    d, ck = 8, 5
    cent = rng.standard_normal((ck, d))
    vals = rng.standard_normal((ck, d))
    lab = rng.permutation(np.repeat(np.arange(ck), 6))
    k = cent[lab]
    v = vals[lab]  # every key/value equals its cluster centroid
    q = rng.standard_normal((30, d))
    qi = q[:3]
    r = eo.pipeline(q, k, v, qi, cent, 3, density=density)
    # zero up to the rounding of the member means (k̄ is a computed mean of equal rows)
    assert np.all(r.e <= 1e-24)
    ref = bf.dense_attention(q, k, v, 1 / math.sqrt(d))
    np.testing.assert_allclose(r.o, ref, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------- P3: covariance identity
@pytest.mark.parametrize("seed", [3, 4])
def test_p3_probe_equals_centroid_quadratic_form(seed):
    q, k, v, qi, ki, it = _head(seed)
    s = 1 / math.sqrt(q.shape[1])
    qc, ql, qn = eo.kmeans(q, qi, it)
    kc, kl, kn = eo.kmeans(k, ki, it)
    e = eo.probe(qc, qn, k, kl, kc, kn, s)
    # E_ab = s^2 q̄_a^T S_b q̄_a with S_b the scatter matrix of cluster b about k̄_b
    ref = np.zeros_like(e)
    for b in range(kc.shape[0]):
        dev = k[kl == b] - kc[b]
        S = dev.T @ dev
        for a in range(qc.shape[0]):
            if qn[a] and kn[b]:
                ref[a, b] = s * s * qc[a] @ S @ qc[a]
    np.testing.assert_allclose(e, ref, rtol=1e-11, atol=1e-13)


# --------------------------------------------------------------------------- P4: singleton key clusters
@pytest.mark.parametrize("density", [0.0, 0.2, 0.5])
def test_p4_singleton_key_clusters_make_compensation_exact(density):
    rng = np.random.default_rng(11)
    q = rng.standard_normal((24, 8))
    k = rng.standard_normal((16, 8))
    v = rng.standard_normal((16, 8))
    r = eo.pipeline(q, k, v, q[:3], k.copy(), 1, density=density)  # C_k = N_k, init = all keys
    assert np.all(r.k_counts == 1)
    ref = bf.dense_attention(q, k, v, 1 / math.sqrt(8))
    np.testing.assert_allclose(r.o, ref, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------- P5: rho = 0
def test_p5_zero_density_is_centroid_attention():
    q, k, v, qi, ki, it = _head(5)
    s = 1 / math.sqrt(q.shape[1])
    r = eo.pipeline(q, k, v, qi, ki, it, density=0.0)
    assert r.exact.sum() == 0 and r.exact_pairs == 0
    nz = r.k_counts > 0
    z = s * q @ r.k_cent[nz].T + np.log(r.k_counts[nz])[None, :]
    w = np.exp(z - z.max(axis=1, keepdims=True))
    ref = (w @ r.v_mean[nz]) / w.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(r.o, ref, rtol=1e-12, atol=1e-12)


def test_p5_one_key_cluster_zero_density_is_mean_of_v():
    q, k, v, qi, ki, it = _head(6)
    r = eo.pipeline(q, k, v, qi, k[:1], it, density=0.0)
    np.testing.assert_allclose(r.o, np.broadcast_to(v.mean(axis=0), r.o.shape), rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------- P6: invariants
@pytest.mark.parametrize("density", [0.0, 0.3, 1.0])
def test_p6_ones_values_and_convex_hull(density):
    q, k, v, qi, ki, it = _head(8)
    r1 = eo.pipeline(q, k, np.ones_like(v), qi, ki, it, density=density)
    np.testing.assert_allclose(r1.o, 1.0, rtol=0, atol=1e-13)
    r = eo.pipeline(q, k, v, qi, ki, it, density=density)
    assert np.all(r.o <= v.max(axis=0) + 1e-12) and np.all(r.o >= v.min(axis=0) - 1e-12)


# --------------------------------------------------------------------------- P7: k-means
@pytest.mark.parametrize("seed,iters", [(0, 1), (1, 3), (2, 6)])
def test_p7_kmeans_matches_scipy_lloyd(seed, iters):
    from scipy.cluster.vq import kmeans2
    rng = np.random.default_rng(seed)
    x = _mixture(rng, 300, 6, 8, 0.4)
    init = x[rng.choice(300, 7, replace=False)]
    c, l, n = eo.kmeans(x, init, iters)
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        c_ref, l_ref = kmeans2(x, init.copy(), iter=iters, minit="matrix", missing="warn")
    np.testing.assert_array_equal(l, l_ref)
    np.testing.assert_allclose(c, c_ref, rtol=1e-13, atol=1e-14)
    assert n.sum() == x.shape[0]
    np.testing.assert_array_equal(n, np.bincount(l_ref, minlength=7))


def test_p7_kmeans_objective_non_increasing_and_labels_are_argmin():
    rng = np.random.default_rng(3)
    x = _mixture(rng, 400, 5, 6, 0.5)
    init = x[rng.choice(400, 6, replace=False)]
    prev = np.inf
    for t in range(1, 7):
        c, l, n = eo.kmeans(x, init, t)
        obj = ((x - c[l]) ** 2).sum()
        assert obj <= prev + 1e-9
        prev = obj
    # labels equal a brute-force argmin against the centroids that produced them
    c_prev, _, _ = eo.kmeans(x, init, 5)
    _, l6, _ = eo.kmeans(x, init, 6)
    dist = ((x[:, None, :] - c_prev[None, :, :]) ** 2).sum(-1)
    np.testing.assert_array_equal(l6, dist.argmin(axis=1))
    # returned centroids are the member means of the returned labels
    c6, l6, n6 = eo.kmeans(x, init, 6)
    for j in range(6):
        if n6[j]:
            np.testing.assert_allclose(c6[j], x[l6 == j].mean(axis=0), rtol=1e-13, atol=1e-14)


# --------------------------------------------------------------------------- P8: permutation
def test_p8_permutation_is_stable_bijection():
    rng = np.random.default_rng(9)
    labels = rng.integers(0, 11, 500)
    labels[labels == 4] = 5  # an empty cluster
    perm, off = eo.permute(labels, 11)
    assert sorted(perm.tolist()) == list(range(500))
    lab_sorted = labels[perm]
    assert np.all(np.diff(lab_sorted) >= 0)
    for c in range(11):
        seg = perm[off[c]:off[c + 1]]
        assert np.all(labels[seg] == c) and np.all(np.diff(seg) > 0)
    np.testing.assert_array_equal(perm, np.argsort(labels, kind="stable"))


# --------------------------------------------------------------------------- P9: routing brute force
@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("density", [0.0, 0.05, 0.25, 0.6, 1.0])
def test_p9_route_matches_literal_greedy(seed, density):
    rng = np.random.default_rng(seed)
    cq, ck = 6, 9
    qn = rng.integers(0, 7, cq)
    kn = rng.integers(0, 9, ck)
    e = rng.exponential(size=(cq, ck))
    e[rng.random((cq, ck)) < 0.2] = 0.0
    e[(qn[:, None] * kn[None, :]) == 0] = 0.0
    nq, nk = int(qn.sum()), int(kn.sum())
    exact, pairs = eo.route(e, qn, kn, nq, nk, density, mode=0)
    # the pages' ratio: block sum of per-entry errors (= |a| E_ab) over |a||b|
    ref, ref_pairs = bf.greedy_route(e * qn[:, None], qn, kn, nq, nk, density)
    np.testing.assert_array_equal(exact, ref)
    assert pairs == ref_pairs
    budget = math.floor(density * nq * nk)
    assert pairs <= budget
    if density == 0.0:
        assert exact.sum() == 0
    # mode 1 = E / (|a||b|)
    exact1, pairs1 = eo.route(e, qn, kn, nq, nk, density, mode=1)
    ref1, ref_pairs1 = bf.greedy_route(e, qn, kn, nq, nk, density)
    np.testing.assert_array_equal(exact1, ref1)
    assert pairs1 == ref_pairs1


# --------------------------------------------------------------------------- P10: token-level brute force
@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("density", [0.0, 0.15, 0.4, 1.0])
@pytest.mark.parametrize("compensate", [True, False])
def test_p10_pipeline_matches_token_level_bruteforce(seed, density, compensate):
    q, k, v, qi, ki, it = _head(seed, nq=64, nk=56)
    s = 1 / math.sqrt(q.shape[1])
    r = eo.pipeline(q, k, v, qi, ki, it, density=density, compensate=compensate)
    # probe: per-entry errors summed over each block equal |a| E_ab
    pe = bf.per_entry_error(r.q_cent, r.q_labels, k, r.k_cent, r.k_labels, s)
    bs = bf.block_sum(pe, r.q_labels, r.k_labels, qi.shape[0], ki.shape[0])
    np.testing.assert_allclose(bs, r.q_counts[:, None] * r.e, rtol=1e-12, atol=1e-12)
    # routing from the per-entry sums
    ex, pairs = bf.greedy_route(bs, r.q_counts, r.k_counts, q.shape[0], k.shape[0], density)
    np.testing.assert_array_equal(ex, r.exact)
    assert pairs == r.exact_pairs
    # v̄ as the per-cluster mean of V
    for b in range(ki.shape[0]):
        if r.k_counts[b]:
            np.testing.assert_allclose(r.v_mean[b], v[r.k_labels == b].mean(axis=0), rtol=1e-13, atol=1e-14)
    if not compensate and r.exact.sum() == 0:
        return
    o, lse = bf.sparse_attention(q, k, v, r.q_labels, r.k_labels, r.k_cent, r.v_mean, r.exact, s,
                                 compensate=compensate)
    valid = np.isfinite(lse)
    np.testing.assert_allclose(r.o[valid], o[valid], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r.lse[valid], lse[valid], rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------- planted mistakes
def test_pins_catch_a_planted_sign_error():
    """A probe with the centroid logit added instead of subtracted fails P3's identity."""
    q, k, v, qi, ki, it = _head(12)
    s = 1 / math.sqrt(q.shape[1])
    qc, ql, qn = eo.kmeans(q, qi, it)
    kc, kl, kn = eo.kmeans(k, ki, it)
    wrong = np.zeros((qc.shape[0], kc.shape[0]))
    for j in range(k.shape[0]):
        b = kl[j]
        wrong[:, b] += (s * qc @ k[j] + s * qc @ kc[b]) ** 2
    e = eo.probe(qc, qn, k, kl, kc, kn, s)
    assert not np.allclose(wrong, e, rtol=1e-6)


# --------------------------------------------------------------------------- weight probes
def _clustered(seed, nq=40, nk=36, d=8, cq=4, ck=5):
    q, k, v, qi, ki, iters = _head(seed, nq, nk, d, cq, ck)
    qc, ql, qn = eo.kmeans(q, qi, iters)
    kc, kl, kn = eo.kmeans(k, ki, iters)
    vm = eo.segment_mean(v, kl, ck)
    return q, k, v, qc, ql, qn, kc, kl, kn, vm


@pytest.mark.parametrize("seed", range(3))
@pytest.mark.parametrize("mode", [1, 2])
def test_weight_probes_match_token_level_bruteforce(seed, mode):
    """Block sums of the token-level estimates, one row per query: every query of
    cluster a uses q̄_a, so the block sum is |a| E[a][b] (SVG-EAR §4.2, §4.3)."""
    q, k, v, qc, ql, qn, kc, kl, kn, vm = _clustered(seed)
    s = 1 / math.sqrt(q.shape[1])
    e = eo.probe_weights(qc, qn, k, kl, kc, kn, v, vm, s, mode)
    per = bf.per_entry_weight_error(qc, ql, k, kc, kl, s, *((v, vm) if mode == 2 else ()))
    blk = bf.block_sum(per, ql, kl, len(qn), len(kn))
    ref = blk / np.maximum(qn, 1)[:, None]
    ref[qn == 0] = 0
    ref[:, kn == 0] = 0
    np.testing.assert_allclose(e, ref, rtol=1e-12, atol=1e-300)


def test_weight_probes_vanish_on_constant_clusters():
    """P2: keys and values equal to their cluster means give zero error."""
    rng = np.random.default_rng(4)
    d, ck, per = 8, 5, 6
    kc = rng.standard_normal((ck, d))
    vc = rng.standard_normal((ck, d))
    kl = np.repeat(np.arange(ck), per).astype(np.int32)
    k, v = kc[kl], vc[kl]
    qc = rng.standard_normal((3, d))
    qn = np.array([4, 0, 2])
    kn = np.full(ck, per)
    for mode in (1, 2):
        e = eo.probe_weights(qc, qn, k, kl, kc, kn, v, vc, 0.3, mode)
        assert np.all(e == 0.0)


def test_value_aware_probe_with_constant_values_scales_the_weight_probe():
    """With v_j = v̄_b in every cluster, ||w v̄ - w̄ v̄||^2 = ||v̄||^2 (w - w̄)^2."""
    q, k, v, qc, ql, qn, kc, kl, kn, vm = _clustered(11)
    vconst = vm[kl]
    s = 0.4
    e1 = eo.probe_weights(qc, qn, k, kl, kc, kn, vconst, vm, s, 1)
    e2 = eo.probe_weights(qc, qn, k, kl, kc, kn, vconst, vm, s, 2)
    np.testing.assert_allclose(e2, e1 * (vm ** 2).sum(axis=1)[None, :], rtol=1e-12, atol=1e-300)


def test_value_aware_probe_with_constant_keys_is_weighted_value_spread():
    """With k_j = k̄_b, w_j = w̄_b and the estimate is w̄_b^2 sum_j ||v_j - v̄_b||^2,
    where w̄_b = e^{s q̄·k̄_b - m}, m the largest logit of the row."""
    rng = np.random.default_rng(12)
    d, ck, per = 6, 4, 5
    kc = rng.standard_normal((ck, d))
    kl = np.repeat(np.arange(ck), per).astype(np.int32)
    k = kc[kl]
    v = rng.standard_normal((ck * per, d))
    vm = eo.segment_mean(v, kl, ck)
    qc = rng.standard_normal((3, d))
    qn = np.ones(3, np.int64)
    kn = np.full(ck, per)
    s = 0.5
    e = eo.probe_weights(qc, qn, k, kl, kc, kn, v, vm, s, 2)
    zc = s * qc @ kc.T
    wbar = np.exp(zc - zc.max(axis=1, keepdims=True))
    spread = np.array([((v[kl == b] - vm[b]) ** 2).sum() for b in range(ck)])
    np.testing.assert_allclose(e, wbar ** 2 * spread[None, :], rtol=1e-12)


def test_weight_probe_small_deviation_limit_is_the_logit_probe():
    """(e^{z} - e^{z̄})^2 = e^{2 z̄} (z - z̄)^2 (1 + O(z - z̄)): for keys within eta
    of their centroids the weight probe tends to w̄_b^2 times the logit probe."""
    rng = np.random.default_rng(13)
    d, ck, per = 8, 4, 6
    base = rng.standard_normal((ck, d))
    kl = np.repeat(np.arange(ck), per).astype(np.int32)
    qc = rng.standard_normal((2, d))
    qn = np.array([3, 5])
    kn = np.full(ck, per)
    s = 0.35
    for eta in (1e-3, 1e-4):
        k = base[kl] + eta * rng.standard_normal((ck * per, d))
        kc = eo.segment_mean(k, kl, ck)
        e_w = eo.probe_weights(qc, qn, k, kl, kc, kn, None, None, s, 1)
        e_l = eo.probe(qc, qn, k, kl, kc, kn, s)
        z = s * qc @ k.T
        zc = s * qc @ kc.T
        wbar2 = np.exp(2 * (zc - z.max(axis=1, keepdims=True)))
        ratio = e_w / (wbar2 * e_l)
        assert np.abs(ratio - 1).max() < 50 * eta


# --------------------------------------------------------------------------- diagnostics
def test_cluster_stats_match_numpy_and_the_kmeans_objective():
    """δ^2 is the k-means objective over N (numpy, written out) and never grows
    over Lloyd iterations; K_max is the largest row norm."""
    rng = np.random.default_rng(31)
    x = _mixture(rng, 300, 16, 7, 0.4)
    init = x[rng.choice(300, 9, replace=False)]
    prev = np.inf
    for it in (1, 2, 4, 8):
        c, l, _ = eo.kmeans(x, init, it)
        ds, km = eo.cluster_stats(x, l, c)
        np.testing.assert_allclose(ds, ((x - c[l]) ** 2).sum(axis=1).mean(), rtol=1e-13)
        np.testing.assert_allclose(km, np.linalg.norm(x, axis=1).max(), rtol=1e-15)
        assert ds <= prev * (1 + 1e-12)
        prev = ds
    # one centroid per row: zero clustering error
    ds, _ = eo.cluster_stats(x[:9], np.arange(9), x[:9])
    assert ds == 0.0


def test_bound_residual_and_normalizer_change_closed_forms():
    assert eo.bound_residual(0.5, 4.0, 1000, 64) == 8 * 0.5 * 16.0 / (1000 * 64)
    lse = np.array([0.0, 1.0, -2.0])
    assert eo.normalizer_change(lse, lse) == 0.0
    # Z doubled for every query: relative change 1; halved: 0.5
    np.testing.assert_allclose(eo.normalizer_change(lse + math.log(2), lse), 1.0, rtol=1e-15)
    np.testing.assert_allclose(eo.normalizer_change(lse - math.log(2), lse), 0.5, rtol=1e-15)


# --------------------------------------------------------------------------- per-query-cluster budgets
def _literal_row_greedy(e, qn, kn, budget):
    exact = np.zeros(e.shape, np.uint8)
    pairs = np.zeros(e.shape[0], np.int64)
    for a in range(e.shape[0]):
        items = sorted(((-e[a, b] / kn[b], b, int(qn[a]) * int(kn[b]))
                        for b in range(e.shape[1]) if qn[a] * kn[b] > 0))
        used = 0
        for _, b, cost in items:
            if used + cost > budget[a]:
                break
            used += cost
            exact[a, b] = 1
        pairs[a] = used
    return exact, pairs


@pytest.mark.parametrize("seed", range(4))
def test_route_rows_matches_literal_greedy_per_row(seed):
    rng = np.random.default_rng(seed)
    cq, ck = 7, 11
    qn = rng.integers(0, 6, cq)
    kn = rng.integers(0, 5, ck)
    e = rng.integers(0, 4, (cq, ck)).astype(float) * kn[None, :]  # many ratio ties
    budget = rng.integers(0, 60, cq)
    exact, pairs = eo.route_rows(e, qn, kn, budget)
    ref, ref_pairs = _literal_row_greedy(e, qn, kn, budget)
    np.testing.assert_array_equal(exact, ref)
    np.testing.assert_array_equal(pairs, ref_pairs)
    cost = qn[:, None] * kn[None, :]
    assert np.all((exact * cost).sum(axis=1) == pairs) and np.all(pairs <= budget)


def test_route_rows_with_one_row_equals_the_global_route():
    """With a single query cluster the per-row walk is the global walk of
    oracle_route under the same budget."""
    rng = np.random.default_rng(9)
    qn = np.array([13])
    kn = rng.integers(0, 9, 30)
    e = rng.random((1, 30)) * kn[None, :]
    for rho in (0.0, 0.1, 0.4, 1.0):
        b = eo.uniform_row_budget(qn, kn.sum(), rho)
        ex_r, pr = eo.route_rows(e, qn, kn, b)
        ex_g, pg = eo.route(e, qn, kn, 13, int(kn.sum()), rho)
        np.testing.assert_array_equal(ex_r, ex_g)
        assert pr[0] == pg


def test_topp_budget_matches_sorted_cumsum_and_special_cases():
    rng = np.random.default_rng(14)
    d, cq, ck = 6, 5, 9
    qc = rng.standard_normal((cq, d))
    kc = rng.standard_normal((ck, d))
    qn = np.array([3, 0, 5, 1, 2])
    kn = np.array([4, 0, 2, 7, 1, 3, 5, 2, 6])
    s = 0.7
    for p in (0.01, 0.3, 0.5, 0.85, 0.999999):
        got = eo.topp_budget(qc, qn, kc, kn, s, p)
        for a in range(cq):
            live = kn > 0
            z = s * qc[a] @ kc[live].T
            w = kn[live] * np.exp(z - z.max())
            order = np.lexsort((np.nonzero(live)[0], -w))
            cum = np.cumsum(w[order]) / w.sum()
            take = int(np.searchsorted(cum, p - 1e-15) + 1)   # smallest prefix reaching p
            keys = kn[live][order][:take].sum()
            assert got[a] == qn[a] * keys
    # p = 1: every non-empty key cluster; equal masses: ceil(p C) clusters
    np.testing.assert_array_equal(eo.topp_budget(qc, qn, kc, kn, s, 1.0), qn * kn.sum())
    flat = eo.topp_budget(np.zeros((1, d)), [1], np.zeros((8, d)), np.ones(8), s, 0.3)
    assert flat[0] == 3
