"""fp64 CPU oracle for reduced attention.

TEST INFRASTRUCTURE ONLY (same rule as ``oracle.rmm``: tests, the smoke check
and the benchmark's CPU-baseline leg only).

Source page: "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product
Reduction for LLM Inference" (technical summary), Metodología › Alcance de
Aplicación: in attention the method reduces the feature dimension of QK^T and,
optionally, the token dimension of PV.  Each reduction is the generic one of
Metodología › Mecanismo Central / Estrategia de Selección with A the
activation-side operand: A = Q for QK^T (contraction over head_dim) and A = P
for PV (contraction over tokens).

READINGS (the page is silent on each; every one is listed in the design notes):
  R1  head_dim indices are scored on Q over all S tokens of one (batch, q-head),
      one index set per (batch, q-head); K is reduced with the same set.
  R2  logits keep the original temperature: scale = 1/sqrt(D) with D the full
      head_dim (the method replaces the product, not the softmax).
  R3  P is the causal softmax of the reduced logits (the two reductions compose).
  R4  one token set per (batch, q-head) over all queries: the literal column
      norm of P, t_j = sum_i P_ij^2.
  R5  O = P[:, I_t] V[I_t, :] with P not renormalised over the kept tokens; a
      query whose causal window holds no kept token gets a zero row.
  R6  grouped-query attention: q-head h reads kv-head floor(h * Hkv / Hq).
"""
from __future__ import annotations

import math

import numpy as np

from .rmm import k_from_rho, column_sq_norms, topk_indices

__all__ = ["attention_head", "reduced_attention", "kv_head_of", "head_dim_selection", "lse_rows",
           "token_scores", "out_rows"]


def kv_head_of(h: int, Hq: int, Hkv: int) -> int:
    """READING R6: kv-head serving q-head h."""
    return (h * Hkv) // Hq


def attention_head(Q, K, V, rho_d: float, rho_t: float, causal: bool = True, scale=None,
                   return_p: bool = False):
    """One (batch, head): Q [S x D], K [S x D], V [S x D] in fp64.

    Returns dict(O [S x D], idx_d [k_d], idx_t [k_t], lse [S], t [S], ssq [D])
    (plus P [S x S] when return_p).
    Steps follow the method's order: score Q's columns, keep the top head_dim
    indices, form the reduced logits, the causal softmax, score P's columns,
    keep the top tokens, form the reduced PV product.
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    S, D = Q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)                      # R2
    # head_dim selection on A = Q (R1)
    ssq = column_sq_norms(Q)
    idx_d = topk_indices(ssq, k_from_rho(rho_d, D))
    # reduced logits S = scale * Q[:, I_d] K[:, I_d]^T
    logits = scale * (Q[:, idx_d] @ K[:, idx_d].T)
    if causal:
        mask = np.tril(np.ones((S, S), dtype=bool))
        logits = np.where(mask, logits, -np.inf)
    # causal softmax (R3)
    mx = np.max(logits, axis=1, keepdims=True)
    e = np.exp(logits - mx)
    z = np.sum(e, axis=1, keepdims=True)
    lse = (mx + np.log(z))[:, 0]
    P = e / z
    # token selection on A = P (R4)
    t = np.einsum("ij,ij->j", P, P)
    idx_t = topk_indices(t, k_from_rho(rho_t, S))
    # reduced PV (R5)
    O = P[:, idx_t] @ V[idx_t, :]
    out = dict(O=O, idx_d=idx_d, idx_t=idx_t, lse=lse, t=t, ssq=ssq)
    if return_p:
        out["P"] = P
    return out


def reduced_attention(Q, K, V, rho_d: float, rho_t: float, causal: bool = True, scale=None,
                      heads=None):
    """Q [B,Hq,S,D], K/V [B,Hkv,S,D] (fp64 values).  ``heads`` optionally
    restricts the work to a list of (b, h) pairs.

    Returns dict of stacked arrays O [B,Hq,S,D], idx_d [B,Hq,k_d],
    idx_t [B,Hq,k_t], lse [B,Hq,S], t [B,Hq,S], ssq [B,Hq,D] (entries of heads
    not computed are left as NaN / -1).
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, Hq, S, D = Q.shape
    Hkv = K.shape[1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    kd = k_from_rho(rho_d, D)
    kt = k_from_rho(rho_t, S)
    out = dict(O=np.full((B, Hq, S, D), np.nan), idx_d=np.full((B, Hq, kd), -1, np.int64),
               idx_t=np.full((B, Hq, kt), -1, np.int64), lse=np.full((B, Hq, S), np.nan),
               t=np.full((B, Hq, S), np.nan), ssq=np.full((B, Hq, D), np.nan))
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in pairs:
        g = kv_head_of(h, Hq, Hkv)
        r = attention_head(Q[b, h], K[b, g], V[b, g], rho_d, rho_t, causal, scale)
        for key in out:
            out[key][b, h] = r[key]
    return out


# ---------------------------------------------------------------- row / column restricted forms
# The same definitions as attention_head, evaluated on chosen query rows or
# key columns only, for sequences whose S x S matrix is too large to hold.
# Each value is computed exactly as in attention_head; only the set of rows
# or columns evaluated is restricted.

def head_dim_selection(Q, rho_d: float):
    """I_d of one (batch, head): top ceil(rho_d D) columns of Q by score (R1)."""
    Q = np.asarray(Q, dtype=np.float64)
    return topk_indices(column_sq_norms(Q), k_from_rho(rho_d, Q.shape[1]))


def lse_rows(Q, K, idx_d, rows, scale=None, chunk: int = 256):
    """lse_i = logsumexp_{j<=i} scale * Q[i, I_d] . K[j, I_d] for i in rows (R2, R3).
    Rows are evaluated `chunk` at a time: one library matmul gives their
    logits against every key up to the chunk's last row, keys past a row's
    position are masked out, and each row's log-sum-exp is then taken alone."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    scale = 1.0 / math.sqrt(Q.shape[1]) if scale is None else scale
    rows = np.asarray(rows, dtype=np.int64)
    Qd, Kd = Q[:, idx_d], K[:, idx_d]
    out = np.empty(len(rows))
    for a in range(0, len(rows), chunk):
        r = rows[a:a + chunk]
        hi = int(r.max()) + 1
        logits = scale * (Qd[r] @ Kd[:hi].T)                       # [rows, keys 0..hi)
        logits[np.arange(hi)[None, :] > r[:, None]] = -np.inf      # causal: j <= i
        mx = logits.max(axis=1)
        out[a:a + len(r)] = mx + np.log(np.sum(np.exp(logits - mx[:, None]), axis=1))
    return out


def token_scores(Q, K, idx_d, lse, cols, scale=None, chunk: int = 256):
    """t_j = sum_{i>=j} P_ij^2 = sum_{i>=j} exp(2 (S_ij - lse_i)) for j in cols (R4),
    given lse for every row.  Columns are evaluated `chunk` at a time: one
    library matmul gives their logits against every query from the chunk's
    first column on, queries before a column's position are masked out, and
    each column's sum is then taken alone."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    scale = 1.0 / math.sqrt(Q.shape[1]) if scale is None else scale
    cols = np.asarray(cols, dtype=np.int64)
    S = Q.shape[0]
    Qd, Kd = Q[:, idx_d], K[:, idx_d]
    out = np.empty(len(cols))
    for a in range(0, len(cols), chunk):
        c = cols[a:a + chunk]
        lo = int(c.min())
        logits = scale * (Qd[lo:] @ Kd[c].T)                       # [queries lo..S, cols]
        e = np.exp(2.0 * (logits - lse[lo:, None]))
        e[np.arange(lo, S)[:, None] < c[None, :]] = 0.0            # causal: i >= j
        out[a:a + len(c)] = e.sum(axis=0)
    return out


def out_rows(Q, K, V, idx_d, lse, idx_t, rows, scale=None):
    """O_i = sum_{j in I_t, j<=i} exp(S_ij - lse_i) V_j for i in rows (R5)."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    scale = 1.0 / math.sqrt(Q.shape[1]) if scale is None else scale
    idx_t = np.asarray(idx_t, dtype=np.int64)
    out = np.zeros((len(rows), V.shape[1]))
    for n, i in enumerate(rows):
        kept = idx_t[idx_t <= i]
        if kept.size:
            p = np.exp(scale * (K[kept][:, idx_d] @ Q[i, idx_d]) - lse[n])
            out[n] = p @ V[kept]
    return out
