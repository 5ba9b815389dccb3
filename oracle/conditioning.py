"""Score-gap conditioning of generated activations (test infrastructure).

TEST INFRASTRUCTURE ONLY (tests and the smoke check; never the product path).

The selected set I is decided by the order of column scores at the k-th /
(k+1)-th boundary.  The oracle ranks fp64 sums; a GPU ranks fp32 sums, whose
relative error is far below 1e-5.  So that both sides must agree on I, the
activation is nudged, deterministically, until every boundary used by the
workload has a relative gap of at least ``rel_gap`` between the last kept and
the first dropped score.  Only the magnitude of single elements of the first
dropped column moves (by one bf16 ulp toward zero, or by a factor 1 - 2^-10
for fp32), so the distribution is unchanged to within rounding noise.

The scores used here are the oracle's own (``oracle.rmm.column_sq_norms``).
"""
from __future__ import annotations

import numpy as np

from .rmm import column_sq_norms, decode

__all__ = ["boundary_gaps", "widen_topk_gaps"]


def boundary_gaps(ss, ks):
    """Relative gap (ss_(k) - ss_(k+1)) / ss_(k+1) at each boundary k (1-based
    rank), with the order (score desc, index asc).  k == d reports +inf."""
    ss = np.asarray(ss, dtype=np.float64)
    d = ss.shape[0]
    order = np.lexsort((np.arange(d), -ss))
    out = {}
    for k in ks:
        if k >= d:
            out[k] = np.inf
            continue
        hi, lo = ss[order[k - 1]], ss[order[k]]
        out[k] = np.inf if lo == 0 and hi > 0 else ((hi - lo) / lo if lo > 0 else 0.0)
    return out, order


def widen_topk_gaps(A, dtype: str, ks, rel_gap: float = 2e-5, max_iters: int = 200000):
    """Return (A', n_nudges): a copy of A (bf16 bits or fp32 [M x d]) whose
    oracle column scores have relative gap >= rel_gap at every boundary in ks."""
    A = np.array(A, copy=True)
    ks = sorted(set(int(k) for k in ks))
    ss = column_sq_norms(decode(A, dtype))
    nudges = 0
    for _ in range(max_iters):
        gaps, order = boundary_gaps(ss, ks)
        bad = [k for k in ks if gaps[k] < rel_gap]
        if not bad:
            return A, nudges
        j = int(order[bad[0]])                    # first dropped column
        col = decode(A[:, j], dtype)
        i = int(np.argmax(np.abs(col)))
        if col[i] == 0.0:
            raise RuntimeError("cannot widen gap: dropped column is all zero")
        if dtype == "bf16":
            A[i, j] = np.uint16(int(A[i, j]) - 1)  # one ulp toward zero (sign-magnitude)
        else:
            A[i, j] = np.float32(A[i, j] * np.float32(1.0 - 2.0 ** -10))
        ss[j] = column_sq_norms(decode(A[:, j:j + 1], dtype))[0]
        nudges += 1
    raise RuntimeError("gap conditioning did not converge")
