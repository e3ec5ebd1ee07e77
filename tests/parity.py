"""Comparison helpers shared by the GPU parity tests.

Top-k sets: equal size; every position in one set but not the other must have
an oracle score within 1e-5 relative of the oracle's cutoff score s_(k) (the
rule the workloads state).  Only where the cutoff is exactly 0 (a row whose
ReLU-clipped keys fill the budget, so a relative band is empty) is a
difference accepted within the fp32 rounding bound of the GPU's score, derived
from the arithmetic: a dot product of n terms accumulated in fp32 is within
gamma_n * sum |q_i k_i| of the exact value, gamma_n = n u / (1 - n u),
u = 2^-24; the weighted ReLU sum adds gamma_H of its absolute terms.
Every check returns the largest |s - s_(k)| / |s_(k)| among the differing
positions, which the tests print.
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


def cutoff_gaps(s, cut, floor_bound=None, rel=1e-5, what=""):
    """Asserts every differing score s sits within rel*|cut| of the cutoff (within
    floor_bound only when cut == 0 exactly); returns the largest relative gap."""
    s = np.asarray(s, np.float64)
    if s.size == 0:
        return 0.0
    gap = np.abs(s - cut)
    if cut == 0.0:
        fb = np.zeros_like(s) if floor_bound is None else np.asarray(floor_bound, np.float64)
        bad = gap > fb
        worst = float(np.max(gap))
    else:
        bad = gap > rel * abs(cut)
        worst = float(np.max(gap) / abs(cut))
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {s.size} differing positions are not "
                           f"within {rel:g} of the cutoff {cut!r}: scores {s[bad][:5]} "
                           f"(relative gaps {(gap[bad] / max(abs(cut), 1e-300))[:5]})")
    return worst


def check_topk_row(g_idx, g_cnt, o_idx, o_cnt, o_cut, score_of, bound_of, rel=1e-5, what=""):
    """g_*/o_*: one row.  score_of(pos array) -> oracle scores; bound_of(pos) -> abs
    fp32 bounds (used only at an exact-0 cutoff).  Returns (differing positions,
    largest relative gap to the cutoff)."""
    assert g_cnt == o_cnt, f"{what}: count {g_cnt} != {o_cnt}"
    gv = g_idx[:g_cnt]
    ov = o_idx[:o_cnt]
    assert (g_idx[g_cnt:] == -1).all(), f"{what}: invalid slots not -1"
    assert (np.diff(gv) > 0).all(), f"{what}: not ascending"
    diff = np.setxor1d(gv, ov)
    if diff.size == 0:
        return 0, 0.0
    s = score_of(diff)
    worst = cutoff_gaps(s, float(o_cut), bound_of(diff) if o_cut == 0.0 else None, rel, what)
    return int(diff.size), worst


def rel_err(g, o):
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    return np.abs(g - o) / np.maximum(1.0, np.abs(o))
