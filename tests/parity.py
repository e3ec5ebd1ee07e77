"""Comparison helpers shared by the GPU parity tests.

Top-k sets: equal size; every position in one set but not the other must have
an oracle score at the cutoff within 1e-5 relative (the rule the workloads
state) plus the fp32 rounding bound of the GPU's score, derived from the
arithmetic: a dot product of n terms accumulated in fp32 is within
gamma_n * sum |q_i k_i| of the exact value, gamma_n = n u / (1 - n u),
u = 2^-24; the weighted ReLU sum adds gamma_H of its absolute terms.
"""
import numpy as np

import oracle

U32 = 2.0 ** -24


def gamma(n):
    return n * U32 / (1 - n * U32)


def indexer_abs_bound(q, w, K):
    """fp32 rounding bound of r = sum_h w_h ReLU(q_h . k) for every key row of K.
    q [H, d], w [H], K [n, d] (float64 arrays of the stored values)."""
    H, d = q.shape
    absdot = np.abs(K) @ np.abs(q).T                     # [n, H]
    dot = K @ q.T
    return (np.abs(w)[None, :] * absdot).sum(1) * gamma(d + 2) + \
        (np.abs(w)[None, :] * np.maximum(dot, 0)).sum(1) * gamma(H + 1)


def check_topk_row(g_idx, g_cnt, o_idx, o_cnt, o_cut, score_of, bound_of, rel=1e-5, what=""):
    """g_*/o_*: one row.  score_of(pos array) -> oracle scores; bound_of(pos) -> abs bounds."""
    assert g_cnt == o_cnt, f"{what}: count {g_cnt} != {o_cnt}"
    gv = g_idx[:g_cnt]
    ov = o_idx[:o_cnt]
    assert (g_idx[g_cnt:] == -1).all(), f"{what}: invalid slots not -1"
    assert (np.diff(gv) > 0).all(), f"{what}: not ascending"
    diff = np.setxor1d(gv, ov)
    if diff.size == 0:
        return 0
    s = score_of(diff)
    b = bound_of(diff)
    tol = rel * abs(o_cut) + 2 * b + 2 * float(np.max(b))
    bad = np.abs(s - o_cut) > tol
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {diff.size} differing positions are "
                           f"not at the cutoff {o_cut!r}: {diff[bad][:5]} scores {s[bad][:5]}")
    return int(diff.size)


def rel_err(g, o):
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    return np.abs(g - o) / np.maximum(1.0, np.abs(o))
