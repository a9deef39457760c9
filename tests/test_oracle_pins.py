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
