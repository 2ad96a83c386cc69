"""Comparison rules between a computed layer output and the oracle's (test
infrastructure only).

Float outputs: per token row, the largest absolute difference divided by the
row's largest reference magnitude (floor 1e-6), maximised over rows. This is
the reading taken of "max relative error" for rows that may contain zeros.
Bound: 2e-2 for bf16 storage, 1e-4 for the fp32 path.
"""
from __future__ import annotations

import numpy as np

TOL_BF16 = 2e-2
TOL_F32 = 1e-4
TOL_GATE = 1e-5

# Router scores: the kernel accumulates bf16 (or fp32) products in fp32, the
# oracle in fp64; scores must agree within LOGIT_ATOL + LOGIT_RTOL * |s|.
LOGIT_ATOL = 1e-4
LOGIT_RTOL = 1e-4


def row_rel_err(y, y_ref, floor=1e-6):
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    if y.shape != y_ref.shape:
        raise ValueError(f"shape {y.shape} != {y_ref.shape}")
    if y.size == 0:
        return 0.0
    num = np.abs(y - y_ref).max(axis=1)
    den = np.maximum(np.abs(y_ref).max(axis=1), floor)
    r = num / den
    if np.isnan(r).any():
        return float("inf")
    return float(r.max())


def tol_for(dtype: str) -> float:
    return TOL_BF16 if dtype == "bf16" else TOL_F32


def outputs_match(y, y_ref, dtype: str) -> bool:
    return row_rel_err(y, y_ref) <= tol_for(dtype)


def permutation_consistent(dest_row, perm_src, offsets, idx, n_kept=None):
    """The combine source-index map is the inverse of the dispatch map on kept
    slots, and each expert segment lists its tokens in ascending order."""
    dest_row = np.asarray(dest_row)
    perm_src = np.asarray(perm_src)
    offsets = np.asarray(offsets)
    idx = np.asarray(idx)
    n = int(offsets[-1]) if n_kept is None else n_kept
    tt, jj = np.nonzero(dest_row >= 0)
    if len(tt) != n:
        return False
    if not np.array_equal(perm_src[dest_row[tt, jj]], tt):
        return False
    e = idx[tt, jj]
    if not ((dest_row[tt, jj] >= offsets[e]) & (dest_row[tt, jj] < offsets[e + 1])).all():
        return False
    for a in range(len(offsets) - 1):
        seg = perm_src[offsets[a]:offsets[a + 1]]
        if seg.size > 1 and not (np.diff(seg) > 0).all():
            return False
    return True


def logits_match(s, s_ref):
    """Finite pattern identical, finite values within the score tolerance."""
    s = np.asarray(s, np.float64)
    s_ref = np.asarray(s_ref, np.float64)
    fin = np.isfinite(s_ref)
    if not np.array_equal(np.isfinite(s), fin):
        return False
    return bool(np.all(np.abs(s[fin] - s_ref[fin]) <= LOGIT_ATOL + LOGIT_RTOL * np.abs(s_ref[fin])))


def gate_bound(gate_ref, s_picked_ref):
    """Allowed |g - g_ref| per slot when the scores themselves may differ by
    the score tolerance. A gate renormalised over the picks is
    g_j = exp(s_j) / sum_i exp(s_i), so dg_j/ds_i = g_j (delta_ij - g_i) and
    |dg_j| <= g_j * 2 * max_i |ds_i|; TOL_GATE covers fp32 exp and division."""
    g = np.asarray(gate_ref, np.float64)
    sp = np.asarray(s_picked_ref, np.float64)
    ds = np.where(np.isfinite(sp), LOGIT_ATOL + LOGIT_RTOL * np.abs(sp), 0.0).max(axis=1, keepdims=True)
    return g * (2.0 * ds + TOL_GATE) + 1e-7


def gates_match(gate, gate_ref, logits_ref, idx_ref):
    sp = np.take_along_axis(np.asarray(logits_ref, np.float64), np.asarray(idx_ref, np.int64), axis=1)
    return bool(np.all(np.abs(np.asarray(gate, np.float64) - gate_ref) <= gate_bound(gate_ref, sp)))


def matrix_rel_err(got, want):
    """max |got - want| / max(max |want|, 1e-6) over one matrix. Used for a
    weight gradient, which is a sum over the tokens routed to one expert: one
    of its rows can be a near-cancelling sum, or (for an expert with a single
    token) a rank-one row scaled by a near-zero factor, so a per-row relative
    error measures rounding of a tiny number; the whole matrix is what an
    update applies, so it is compared against its own largest element."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    if want.size == 0:
        return 0.0
    return float(np.abs(got - want).max() / max(np.abs(want).max(), 1e-6))


def vector_rel_err(got, want):
    """max |got - want| / max(max |want|, 1e-6) over one vector (a whole row
    or column of a weight gradient). A wrong sign, a zero or a missing term of
    the sum changes the vector by the order of its own largest element."""
    return matrix_rel_err(np.asarray(got, np.float64).reshape(1, -1), np.asarray(want, np.float64).reshape(1, -1))
