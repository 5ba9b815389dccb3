"""fp64 CPU oracle for the reduced matrix product.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this module.  The CUDA path never
calls it, links it or reads anything it produced at run time.

Source page: "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product
Reduction for LLM Inference" (technical summary, gist.science; Spanish and
Chinese editions carry the same text).  Section names below are the Spanish
edition's ("Metodología" = Methodology).

Everything here is the plain definition written out in fp64 on the exact
stored input values; a library matmul serves as one step.  Readings of points
the page leaves open are marked READING.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = ["k_from_rho", "column_sq_norms", "column_norms", "topk_indices",
           "reduced_matmul", "dense_matmul", "rmm", "decode", "dequantize_w8",
           "reduced_matmul_w8", "rmm_w8"]


def decode(x, dtype: str) -> np.ndarray:
    """Exact fp64 values of a stored input: dtype "bf16" (uint16 bits) or "f32"."""
    if dtype == "bf16":
        b = np.ascontiguousarray(np.asarray(x, dtype=np.uint16))
        return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if dtype in ("f32", "f64"):
        return np.asarray(x, dtype=np.float64)
    raise ValueError(f"unknown dtype {dtype}")


def k_from_rho(rho: float, d: int) -> int:
    """Number of kept contraction indices, k = ceil(rho * d).

    Metodología › Estrategia de Selección: the top-k indices are kept with
    k = ceil(rho d), rho a user retention ratio.
    READING: rho must lie in (0, 1]; the product rho*d is formed in fp64 and a
    guard of 1e-9*d absorbs representation error (0.3*10 = 3.0000000000000004
    gives k = 3, not 4); the result is clamped to [1, d].
    """
    if not (isinstance(d, (int, np.integer)) and d >= 1):
        raise ValueError("d must be a positive integer")
    if not (0.0 < float(rho) <= 1.0) or math.isnan(rho):
        raise ValueError("rho must lie in (0, 1]")
    k = math.ceil(float(rho) * d - 1e-9 * d)
    return int(min(max(k, 1), d))


def column_sq_norms(A) -> np.ndarray:
    """ss_j = sum_i A_ij^2 in fp64, one value per column of A [M x d].

    Metodología › Estrategia de Selección: the importance score of feature j is
    the column norm s_j = ||A[:, j]||_2.  Ranking by ss_j = s_j^2 is the same
    ranking (the square is monotone on s >= 0).
    """
    A = np.asarray(A, dtype=np.float64)
    if A.ndim != 2:
        raise ValueError("A must be 2-D")
    if not np.all(np.isfinite(A)):
        raise ValueError("non-finite activation (not defined by the method)")
    return np.einsum("ij,ij->j", A, A)


def column_norms(A) -> np.ndarray:
    """s_j = ||A[:, j]||_2 (Metodología › Estrategia de Selección)."""
    return np.sqrt(column_sq_norms(A))


def topk_indices(scores, k: int) -> np.ndarray:
    """The k indices with the largest scores, returned in ascending order.

    Metodología › Estrategia de Selección: keep the top-k indices by score.
    READING (the page fixes neither): ties are broken toward the lowest index;
    the kept set is reported in ascending index order.  Implemented as a stable
    sort on (-score, index).
    """
    s = np.asarray(scores, dtype=np.float64)
    if s.ndim != 1:
        raise ValueError("scores must be 1-D")
    d = s.shape[0]
    if not (1 <= k <= d):
        raise ValueError("need 1 <= k <= d")
    if not np.all(np.isfinite(s)):
        raise ValueError("non-finite score")
    order = np.lexsort((np.arange(d), -s))  # primary key -s, secondary index
    return np.sort(order[:k]).astype(np.int64)


def reduced_matmul(A, B, idx) -> np.ndarray:
    """Y = A[:, I] B[I, :] in fp64.

    Metodología › Mecanismo Central: instead of AB the method computes the
    reduced product A_{:,I} B_{I,:} over the kept subset I of the shared
    contraction dimension.
    """
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    idx = np.asarray(idx, dtype=np.int64)
    if A.shape[1] != B.shape[0]:
        raise ValueError("contraction dimensions differ")
    return A[:, idx] @ B[idx, :]


def dense_matmul(A, B) -> np.ndarray:
    """Y = AB in fp64 (the product the method replaces; Metodología)."""
    return np.asarray(A, dtype=np.float64) @ np.asarray(B, dtype=np.float64)


def rmm(A, B, rho: float):
    """Whole path: scores -> top-k -> reduced product.  Returns (Y, I, ss)."""
    A = np.asarray(A, dtype=np.float64)
    ss = column_sq_norms(A)
    k = k_from_rho(rho, A.shape[1])
    idx = topk_indices(ss, k)
    return reduced_matmul(A, B, idx), idx, ss


def dequantize_w8(Bq, scale) -> np.ndarray:
    """The weight an int8 matrix stands for: B[j, n] = Bq[j, n] * scale[n], fp64.

    Resultados Experimentales › Compatibilidad: the method is reported to work
    with INT8 weight quantisation.  READING (the page names no scheme):
    symmetric weight-only quantisation with one scale per output column n of
    the [d x N] weight, no zero point.
    """
    q = np.asarray(Bq)
    if q.dtype != np.int8:
        raise ValueError("Bq must be int8")
    s = np.asarray(scale, dtype=np.float64)
    if s.ndim != 1 or s.shape[0] != q.shape[1]:
        raise ValueError("one scale per column of Bq")
    if not np.all(np.isfinite(s)):
        raise ValueError("non-finite scale")
    return q.astype(np.float64) * s[None, :]


def reduced_matmul_w8(A, Bq, scale, idx) -> np.ndarray:
    """Y = A[:, I] B[I, :] with B the int8 weight's dequantised values, fp64.

    Metodología › Mecanismo Central (the reduced product) applied to the
    weight of Resultados Experimentales › Compatibilidad (see dequantize_w8).
    The rows are restricted to I first, then dequantised.
    """
    idx = np.asarray(idx, dtype=np.int64)
    q = np.asarray(Bq)
    A = np.asarray(A, dtype=np.float64)
    if A.shape[1] != q.shape[0]:
        raise ValueError("contraction dimensions differ")
    return A[:, idx] @ dequantize_w8(q[idx, :], scale)


def rmm_w8(A, Bq, scale, rho: float):
    """Whole path with an int8 weight: scores of A -> top-k -> reduced product.

    The selection reads only the activation (Metodología › Estrategia de
    Selección), so it is the same index set as for any other weight.
    Returns (Y, I, ss).
    """
    A = np.asarray(A, dtype=np.float64)
    ss = column_sq_norms(A)
    k = k_from_rho(rho, A.shape[1])
    idx = topk_indices(ss, k)
    return reduced_matmul_w8(A, Bq, scale, idx), idx, ss
