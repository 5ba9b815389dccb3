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

__all__ = ["attention_head", "reduced_attention", "kv_head_of"]


def kv_head_of(h: int, Hq: int, Hkv: int) -> int:
    """READING R6: kv-head serving q-head h."""
    return (h * Hkv) // Hq


def attention_head(Q, K, V, rho_d: float, rho_t: float, causal: bool = True, scale=None):
    """One (batch, head): Q [S x D], K [S x D], V [S x D] in fp64.

    Returns dict(O [S x D], idx_d [k_d], idx_t [k_t], lse [S], t [S], ssq [D]).
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
    return dict(O=O, idx_d=idx_d, idx_t=idx_t, lse=lse, t=t, ssq=ssq)


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
