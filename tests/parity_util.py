"""Helpers for the GPU parity tests: moving seeded inputs to the device and
the comparison rules (tolerances) of each step."""
from __future__ import annotations

import math

import numpy as np

# Attention given the same mask (compared with the fp64 oracle):
#   bf16 inputs, fp32 accumulation: max-abs 2e-2 and relative L2 5e-3
#   fp32 inputs:                    max-abs 1e-4
ATTN_TOL = {"bf16": (2e-2, 5e-3), "f32": (1e-4, 1e-4)}
# Natural-log normalizer (lse).  bf16 inputs: the exact logits s q·k are bf16
# products summed in fp32 (relative ~1e-6), and the compensated logits use the
# key centroids as a bf16 hi + lo pair (16 significant bits, so s q·k̄ moves by
# about s 2^-17 sqrt(sum_k q_k^2 k̄_k^2) ~ 1e-5 at d = 128); the sum l is fp32.
# 2e-3 leaves room for the ex2.approx exponent and for sums of many terms.
# fp32 inputs run in fp32 throughout.
LSE_TOL = {"bf16": 2e-3, "f32": 1e-5}
# k-means / route ties: a differing label or block is allowed only within 1e-6 relative
TIE_REL = 1e-6


def torch_dtype(name):
    import torch
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def dev(x, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def host(t):
    import torch
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.cpu().numpy()


def attention_errors(o_gpu, o_ref):
    o_gpu = np.asarray(o_gpu, np.float64)
    o_ref = np.asarray(o_ref, np.float64)
    max_abs = float(np.abs(o_gpu - o_ref).max())
    rel_l2 = float(np.linalg.norm(o_gpu - o_ref) / max(np.linalg.norm(o_ref), 1e-300))
    return max_abs, rel_l2


def assert_attention_close(o_gpu, o_ref, dtype):
    max_abs, rel_l2 = attention_errors(o_gpu, o_ref)
    tol_abs, tol_rel = ATTN_TOL[dtype]
    assert max_abs <= tol_abs and rel_l2 <= tol_rel, (max_abs, rel_l2)
    return max_abs, rel_l2


def assert_labels_exact_or_tie(x, cent, lab_gpu, lab_ref):
    """Labels must match; a mismatch is allowed only at a distance tie within
    1e-6 of (|x|^2 + |c|^2), both distances in fp64 against the same centroids."""
    x = np.asarray(x, np.float64)
    cent = np.asarray(cent, np.float64)
    bad = np.nonzero(lab_gpu != lab_ref)[0]
    for i in bad:
        dg = ((x[i] - cent[lab_gpu[i]]) ** 2).sum()
        dr = ((x[i] - cent[lab_ref[i]]) ** 2).sum()
        scale = (x[i] ** 2).sum() + (cent[lab_ref[i]] ** 2).sum()
        assert abs(dg - dr) <= TIE_REL * scale, (i, lab_gpu[i], lab_ref[i], dg, dr)
    return len(bad)


def route_ratio(e, qn, kn, mode):
    cost = qn[:, None].astype(np.float64) * kn[None, :].astype(np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(cost > 0, e / (kn[None, :] if mode == 0 else cost), np.nan)
    return r


def assert_route_exact_or_tie(exact_gpu, exact_ref, e, qn, kn, mode):
    """Exact masks must match; a differing block is allowed only if its ratio is
    within 1e-6 (relative) of the ratio of the oracle's cut."""
    diff = np.argwhere(exact_gpu != exact_ref)
    if len(diff) == 0:
        return 0
    r = route_ratio(np.asarray(e, np.float64), np.asarray(qn), np.asarray(kn), mode)
    sel = r[exact_ref.astype(bool)]
    cut = sel.min() if sel.size else np.nanmax(r)
    for a, b in diff:
        assert abs(r[a, b] - cut) <= TIE_REL * max(abs(cut), 1e-300), (a, b, r[a, b], cut)
    return len(diff)


def scale_of(d):
    return 1.0 / math.sqrt(d)
