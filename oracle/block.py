"""fp64 CPU oracle for the block driver: products that share one activation
share one selection, and a gated MLP block with every product reduced.

TEST INFRASTRUCTURE ONLY (same rule as ``oracle.rmm``: tests, the smoke check
and the benchmark's CPU-baseline leg only).

Source page: "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product
Reduction for LLM Inference" (technical summary).  Metodología › Mecanismo
Central: I is chosen from the activation A alone, so products with the same A
(q, k, v of an attention input; up and gate of an MLP input) have the same I.
Contribuciones Clave › Perspectivas Mecanísticas: components differ in how
much reduction they tolerate, hence one rho per component.

READINGS (listed in the design notes):
  B1  intermediate activations (the up and gate outputs, H) are stored as
      bf16, rounded to nearest even, as in a bf16 model;
  B2  SiLU(g) = g / (1 + e^-g), the gated activation H = SiLU(G) * U;
  B3  the down projection's selection is scored on the stored H.
"""
from __future__ import annotations

import math

import numpy as np

from .rmm import k_from_rho, column_sq_norms, topk_indices, reduced_matmul

__all__ = ["matmul_shared", "round_bf16", "silu_mul_bf16", "mlp_block"]


def matmul_shared(A, Bs, rho: float):
    """Y_i = A[:, I] B_i[I, :] for every weight B_i, with one I = top-k of A's
    column scores.  Returns ([Y_i], I, ss)."""
    A = np.asarray(A, dtype=np.float64)
    ss = column_sq_norms(A)
    idx = topk_indices(ss, k_from_rho(rho, A.shape[1]))
    return [reduced_matmul(A, B, idx) for B in Bs], idx, ss


def round_bf16(x) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value (8 significant bits, ties to
    even); returns the rounded values in fp64 (B1).  Finite normal range only."""
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite value")
    m, e = np.frexp(x)                      # x = m 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def silu_mul_bf16(G, U) -> np.ndarray:
    """H = bf16(SiLU(G) * U) with SiLU(g) = g / (1 + e^-g) in fp64 (B1, B2)."""
    G = np.asarray(G, dtype=np.float64)
    U = np.asarray(U, dtype=np.float64)
    return round_bf16(G / (1.0 + np.exp(-G)) * U)


def mlp_block(X, W_up, W_gate, W_down, rho_up: float, rho_down: float):
    """Gated MLP block with every product reduced.

    U, G = X[:, I] W_up[I, :], X[:, I] W_gate[I, :] with one I from X (rho_up),
    both stored as bf16 (B1); H = bf16(SiLU(G) * U) (B2); Y = H[:, J]
    W_down[J, :] with J the top ceil(rho_down d_ff) columns of H by score (B3).
    Returns dict(Y, I, J, H, ssH)."""
    X = np.asarray(X, dtype=np.float64)
    (Uf, Gf), I, _ = matmul_shared(X, [W_up, W_gate], rho_up)
    H = silu_mul_bf16(round_bf16(Gf), round_bf16(Uf))
    ssH = column_sq_norms(H)
    J = topk_indices(ssH, k_from_rho(rho_down, H.shape[1]))
    Y = reduced_matmul(H, W_down, J)
    return dict(Y=Y, I=I, J=J, H=H, ssH=ssH)
