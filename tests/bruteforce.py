"""Token-level brute force of SVG-EAR, written independently of the C++ oracle.

Used only by the CPU pin tests on tiny inputs.  It follows the token-level
statement of the method (SVG-EAR §4.1 routing mask M in {0,1}^{N_q x N_k},
§4.3 Linear Compensation): it materialises the whole N_q x N_k logit matrix,
with the exact logit s q_i·k_j where M=1 and the compensated logit
s q_i·k̄_{b(j)} (value v̄_{b(j)}) where M=0, and takes one softmax over each
row.  The probe is the per-entry estimate eps_ij^2 = (s q̄_i·k_j - s q̄_i·k̄_j)^2
summed over each block, and routing is a literal greedy walk in Python.
"""
from __future__ import annotations

import math

import numpy as np


def token_mask(exact, q_labels, k_labels):
    """Expand the block mask to M[i, j] = exact[label(q_i), label(k_j)]."""
    return np.asarray(exact, bool)[np.asarray(q_labels)[:, None], np.asarray(k_labels)[None, :]]


def sparse_attention(q, k, v, q_labels, k_labels, k_cent, v_cent, exact, scale, compensate=True):
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    M = token_mask(exact, q_labels, k_labels)
    kbar = np.asarray(k_cent, np.float64)[k_labels]      # per-token key centroid  (K̄)
    vbar = np.asarray(v_cent, np.float64)[k_labels]      # per-token value mean    (V̄)
    exact_logits = scale * q @ k.T
    comp_logits = scale * q @ kbar.T
    z = np.where(M, exact_logits, comp_logits if compensate else -np.inf)
    m = z.max(axis=1, keepdims=True)
    with np.errstate(invalid="ignore"):  # rows with no term at all give NaN, callers mask them
        w = np.exp(z - m)
    # each key j contributes w_ij times v_j (exact) or v̄_j (compensated)
    out = (w * M) @ v + (w * ~M) @ vbar if compensate else (w * M) @ v
    L = w.sum(axis=1, keepdims=True)
    return out / L, (m + np.log(L))[:, 0]


def dense_attention(q, k, v, scale):
    """Textbook softmax(s Q K^T) V in fp64."""
    z = scale * np.asarray(q, np.float64) @ np.asarray(k, np.float64).T
    z -= z.max(axis=1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=1, keepdims=True)
    return p @ np.asarray(v, np.float64)


def per_entry_error(q_cent, q_labels, k, k_cent, k_labels, scale):
    """eps_ij^2 for every (query i, key j), with q̄_i standing in for q_i."""
    qbar = np.asarray(q_cent, np.float64)[q_labels]
    kbar = np.asarray(k_cent, np.float64)[k_labels]
    exact = scale * qbar @ np.asarray(k, np.float64).T
    approx = scale * qbar @ kbar.T
    return (exact - approx) ** 2


def block_sum(per_entry, q_labels, k_labels, c_q, c_k):
    out = np.zeros((c_q, c_k))
    np.add.at(out, (np.asarray(q_labels)[:, None], np.asarray(k_labels)[None, :]), per_entry)
    return out


def greedy_route(block_err_sum, q_counts, k_counts, n_q, n_k, density):
    """Literal greedy walk: ratio = (sum of per-entry errors in block) / (|q_c| |k_c|)."""
    budget = math.floor(density * float(n_q * n_k))
    c_q, c_k = block_err_sum.shape
    items = []
    for a in range(c_q):
        for b in range(c_k):
            cost = int(q_counts[a]) * int(k_counts[b])
            if cost:
                items.append((-block_err_sum[a, b] / cost, a * c_k + b, cost))
    items.sort()
    exact = np.zeros((c_q, c_k), np.uint8)
    used = 0
    for _, idx, cost in items:
        if used + cost > budget:
            break
        used += cost
        exact[idx // c_k, idx % c_k] = 1
    return exact, used


def per_entry_weight_error(q_cent, q_labels, k, k_cent, k_labels, scale, v=None, v_cent=None):
    """Unnormalized-weight estimates for every (query i, key j), with q̄_i for
    q_i and each query cluster's weights taken relative to e^{m}, m the largest
    logit s q̄_i·k_j of its row: (w_ij - w̄_ij)^2, or with values
    ||w_ij v_j - w̄_ij v̄_j||^2."""
    qbar = np.asarray(q_cent, np.float64)[q_labels]
    kbar = np.asarray(k_cent, np.float64)[k_labels]
    z = scale * qbar @ np.asarray(k, np.float64).T
    zc = scale * qbar @ kbar.T
    m = z.max(axis=1, keepdims=True)
    w, wc = np.exp(z - m), np.exp(zc - m)
    if v is None:
        return (w - wc) ** 2
    vv = np.asarray(v, np.float64)
    vb = np.asarray(v_cent, np.float64)[k_labels]
    diff = w[:, :, None] * vv[None, :, :] - wc[:, :, None] * vb[None, :, :]
    return (diff ** 2).sum(axis=2)
