"""fp64 CPU oracle for reduced attention at decode time (one new query token
per sequence over a cache of L keys and values).

TEST INFRASTRUCTURE ONLY (same rule as ``oracle.rmm``: tests, the smoke check
and the benchmark's CPU-baseline leg only).

Source page: "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product
Reduction for LLM Inference" (technical summary).  Metodología › Alcance de
Aplicación: the feature dimension of QK^T and the token dimension of PV are
reduced; Resultados Experimentales: the method stays stable in autoregressive
generation.  The page does not describe the decode step itself; the readings
below apply the prefill readings of ``oracle.attention`` to one query row.

READINGS (listed in the design notes):
  D1  the new token's query attends to all L cached tokens (its own key and
      value are the cache's last row); no mask inside the cache.
  D2  head_dim is scored on the single query row (R1 with one token):
      ss_c = q_c^2; I_d = top ceil(rho_d D), lowest index on ties.
  D3  token scores are the column norms of the single-row P (R4 with one
      query): t_j = P_j^2; I_t = top ceil(rho_t L), lowest index on ties.
  D4  R2 (scale 1/sqrt(D) of the full head_dim), R5 (no renormalisation of P
      over I_t) and R6 (q-head h reads kv-head floor(h Hkv / Hq)) as in prefill.
"""
from __future__ import annotations

import math

import numpy as np

from .rmm import k_from_rho, column_sq_norms, topk_indices
from .attention import kv_head_of

__all__ = ["decode_attention_head", "decode_attention"]


def decode_attention_head(q, K, V, rho_d: float, rho_t: float, scale=None):
    """One (sequence, q-head): q [D], K [L x D], V [L x D] in fp64.

    Returns dict(O [D], idx_d [k_d], idx_t [k_t], lse (scalar), logits [L],
    t [L], ssq [D]).  Steps in the method's order: score the query's
    head_dim entries, keep the top ones, form the reduced logits over the
    cache, the softmax, score the tokens by P_j^2, keep the top tokens, form
    the reduced PV product.
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    L, D = K.shape
    if q.shape != (D,) or V.shape[0] != L:
        raise ValueError("shapes: q [D], K [L x D], V [L x Dv]")
    if scale is None:
        scale = 1.0 / math.sqrt(D)                                    # D4 (R2)
    ssq = column_sq_norms(q[None, :])                                 # D2
    idx_d = topk_indices(ssq, k_from_rho(rho_d, D))
    logits = scale * (K[:, idx_d] @ q[idx_d])                         # D1
    mx = np.max(logits)
    e = np.exp(logits - mx)
    z = np.sum(e)
    lse = mx + np.log(z)
    P = e / z
    t = P * P                                                         # D3
    idx_t = topk_indices(t, k_from_rho(rho_t, L))
    O = P[idx_t] @ V[idx_t, :]                                        # D4 (R5)
    return dict(O=O, idx_d=idx_d, idx_t=idx_t, lse=lse, logits=logits, t=t, ssq=ssq)


def decode_attention(q, K, V, L: int, rho_d: float, rho_t: float, scale=None, heads=None):
    """q [B,Hq,D], caches K/V [B,Hkv,Lmax,D] holding L valid tokens (fp64
    values).  ``heads`` optionally restricts the work to (b, h) pairs.

    Returns dict of stacked arrays O [B,Hq,D], idx_d [B,Hq,k_d],
    idx_t [B,Hq,k_t], lse [B,Hq], logits [B,Hq,L] (entries of heads not
    computed are NaN / -1).
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    B, Hq, D = q.shape
    Hkv = K.shape[1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    if not (1 <= L <= K.shape[2]):
        raise ValueError("need 1 <= L <= cache capacity")
    kd, kt = k_from_rho(rho_d, D), k_from_rho(rho_t, L)
    out = dict(O=np.full((B, Hq, V.shape[3]), np.nan), idx_d=np.full((B, Hq, kd), -1, np.int64),
               idx_t=np.full((B, Hq, kt), -1, np.int64), lse=np.full((B, Hq), np.nan),
               logits=np.full((B, Hq, L), np.nan))
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in pairs:
        g = kv_head_of(h, Hq, Hkv)
        r = decode_attention_head(q[b, h], K[b, g, :L], V[b, g, :L], rho_d, rho_t, scale)
        for key in out:
            out[key][b, h] = r[key]
    return out
