"""Pins for the fp64 reduced-matmul oracle against facts fixed by the page and
by mathematics: closed forms, brute force over all subsets, the dense special
case, an error bound and its tight construction.  CPU only."""
import itertools
import math

import numpy as np
import pytest

import oracle
from oracle import rmm as O
import workloads as W


# ------------------------------------------------------------------ k = ceil(rho d)

@pytest.mark.parametrize("rho,d,k", [
    (0.5, 4096, 2048), (0.7, 4096, 2868), (0.8, 4096, 3277), (1.0, 4096, 4096),
    (0.5, 14336, 7168), (0.8, 14336, 11469), (1.0, 14336, 14336),
    (0.8, 8192, 6554), (0.8, 28672, 22938), (0.5, 8192, 4096), (0.5, 128, 64),
    (0.5, 256, 128), (0.3, 10, 3), (0.51, 100, 51), (0.501, 1000, 501),
    (1e-9, 100, 1), (0.5, 1, 1), (0.5, 32768, 16384), (0.999, 7, 7), (0.15, 7, 2),
])
def test_k_from_rho_closed_form(rho, d, k):
    assert O.k_from_rho(rho, d) == k


@pytest.mark.parametrize("rho", [0.0, -0.1, 1.0000001, float("nan")])
def test_k_from_rho_rejects(rho):
    with pytest.raises(ValueError):
        O.k_from_rho(rho, 16)


# ------------------------------------------------------------------ scores

def test_column_scores_closed_form():
    A = np.array([[3.0, 0.0, 1.0, -2.0], [4.0, 0.0, -1.0, 0.5]])
    np.testing.assert_array_equal(O.column_sq_norms(A), [25.0, 0.0, 2.0, 4.25])
    np.testing.assert_allclose(O.column_norms(A), [5.0, 0.0, math.sqrt(2), math.sqrt(4.25)])


def test_column_scores_rejects_nonfinite():
    with pytest.raises(ValueError):
        O.column_sq_norms(np.array([[1.0, np.inf]]))


def test_bf16_decode_known_values():
    bits = np.array([0x3F80, 0xBF80, 0x4000, 0x0000, 0x8000, 0x3F81, 0x7F7F], np.uint16)
    vals = O.decode(bits, "bf16")
    np.testing.assert_array_equal(vals[:5], [1.0, -1.0, 2.0, 0.0, -0.0])
    assert vals[5] == 1.0 + 2.0 ** -7
    assert vals[6] == (2.0 - 2.0 ** -7) * 2.0 ** 127


# ------------------------------------------------------------------ top-k

def brute_topk(s, k):
    """All C(d,k) subsets: the maximal kept sum; among maximisers the
    lexicographically smallest ascending tuple (the lowest-index tie rule)."""
    best, best_set = None, None
    for c in itertools.combinations(range(len(s)), k):  # lexicographic order
        v = sum(s[j] for j in c)
        if best is None or v > best:
            best, best_set = v, c
    return list(best_set)


@pytest.mark.parametrize("trial", range(12))
def test_topk_bruteforce_small(trial):
    rng = np.random.default_rng(100 + trial)
    d = int(rng.integers(3, 13))
    # integer-valued scores with many ties, so the tie rule is exercised
    s = rng.integers(0, 5, size=d).astype(np.float64)
    for k in range(1, d + 1):
        assert list(O.topk_indices(s, k)) == brute_topk(list(s), k), (s, k)


@pytest.mark.parametrize("trial", range(6))
def test_topk_bruteforce_distinct(trial):
    """c0-distributed slices of up to 16 columns: exact sums of exact squares."""
    inp = W.tiny_fp32(seed=trial)
    A = O.decode(inp.A, "f32")
    cols = np.random.default_rng(trial).choice(A.shape[1], size=14, replace=False)
    ss = O.column_sq_norms(A[:, cols])
    for k in (1, 3, 7, 13, 14):
        assert list(O.topk_indices(ss, k)) == brute_topk(list(ss), k)


def test_topk_ties_special_cases():
    assert list(O.topk_indices(np.ones(10), 4)) == [0, 1, 2, 3]
    assert list(O.topk_indices(np.zeros(7), 7)) == list(range(7))
    s = np.array([0.0, 5.0, 1.0, 5.0, 5.0, 2.0])
    assert list(O.topk_indices(s, 1)) == [1]
    assert list(O.topk_indices(s, 2)) == [1, 3]
    assert list(O.topk_indices(s, 4)) == [1, 3, 4, 5]
    assert list(O.topk_indices(s, 6)) == list(range(6))
    with pytest.raises(ValueError):
        O.topk_indices(s, 0)
    with pytest.raises(ValueError):
        O.topk_indices(s, 7)


def test_topk_certificate_c0():
    inp = W.tiny_fp32(0)
    A = O.decode(inp.A, "f32")
    ss = O.column_sq_norms(A)
    k = O.k_from_rho(0.5, A.shape[1])
    idx = O.topk_indices(ss, k)
    rest = np.setdiff1d(np.arange(A.shape[1]), idx)
    assert len(idx) == k and np.all(np.diff(idx) > 0)
    assert ss[idx].min() >= ss[rest].max()


# ------------------------------------------------------------------ reduced product

def test_identity_weight_closed_form():
    """With B = I_d the reduced product is A with dropped columns zeroed."""
    rng = np.random.default_rng(7)
    A = rng.standard_normal((9, 12)) * np.arange(1, 13)[None, :]
    Y, idx, _ = O.rmm(A, np.eye(12), 0.5)
    expect = np.zeros_like(A)
    expect[:, 6:] = A[:, 6:]          # column norms grow with the column index
    np.testing.assert_array_equal(idx, np.arange(6, 12))
    np.testing.assert_array_equal(Y, expect)


def test_permutation_weight_closed_form():
    """B a permutation: Y[:, p(j)] = A[:, j] for kept j, zero elsewhere."""
    rng = np.random.default_rng(8)
    d = 10
    A = rng.standard_normal((5, d)) * (d - np.arange(d))[None, :]
    p = rng.permutation(d)
    B = np.zeros((d, d))
    B[np.arange(d), p] = 1.0
    Y, idx, _ = O.rmm(A, B, 0.3)
    np.testing.assert_array_equal(idx, [0, 1, 2])
    expect = np.zeros((5, d))
    for j in idx:
        expect[:, p[j]] = A[:, j]
    np.testing.assert_array_equal(Y, expect)


def test_rho_one_is_dense():
    inp = W.tiny_fp32(0)
    A, B = O.decode(inp.A, "f32"), O.decode(inp.B, "f32")
    Y, idx, _ = O.rmm(A, B, 1.0)
    np.testing.assert_array_equal(idx, np.arange(A.shape[1]))
    np.testing.assert_allclose(Y, O.dense_matmul(A, B), rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("rho", [0.25, 0.5, 0.8])
def test_error_bound(rho):
    """||AB - A_I B_I||_F <= ||A_{I^c}||_F ||B_{I^c}||_2 (Cauchy-Schwarz +
    submultiplicativity), spectral norm from LAPACK's SVD."""
    inp = W.tiny_fp32(0)
    A, B = O.decode(inp.A, "f32"), O.decode(inp.B, "f32")
    Y, idx, _ = O.rmm(A, B, rho)
    rest = np.setdiff1d(np.arange(A.shape[1]), idx)
    err = np.linalg.norm(O.dense_matmul(A, B) - Y)
    bound = np.linalg.norm(A[:, rest]) * np.linalg.norm(B[rest, :], 2)
    assert err <= bound * (1 + 1e-9)
    assert err <= np.linalg.norm(A[:, rest]) * np.linalg.norm(B[rest, :]) * (1 + 1e-9)


def test_minimax_tight_construction():
    """Worst case over ||B||_2 <= 1: with orthonormal rows on I^c and zero rows
    on I the error equals ||A_{I^c}||_F exactly (N = d - k)."""
    inp = W.tiny_fp32(0)
    A = O.decode(inp.A, "f32")
    d = A.shape[1]
    k = O.k_from_rho(0.5, d)
    idx = O.topk_indices(O.column_sq_norms(A), k)
    rest = np.setdiff1d(np.arange(d), idx)
    q, _ = np.linalg.qr(np.random.default_rng(3).standard_normal((d - k, d - k)))
    Bstar = np.zeros((d, d - k))
    Bstar[rest, :] = q
    Y, idx2, _ = O.rmm(A, Bstar, 0.5)
    np.testing.assert_array_equal(idx, idx2)
    err = np.linalg.norm(O.dense_matmul(A, Bstar) - Y)
    assert abs(err - np.linalg.norm(A[:, rest])) <= 1e-12 * np.linalg.norm(A)
    assert np.linalg.norm(Y) == 0.0


def test_topk_minimises_worst_case_over_subsets():
    """Top-k by column norm minimises ||A_{I^c}||_F, the worst-case error over
    unit-spectral-norm B (Metodología › Base Teórica): brute force over all
    subsets at d = 12, and against 100 random subsets at d = 256."""
    rng = np.random.default_rng(4)
    A = rng.standard_normal((6, 12)) * rng.uniform(0.1, 3, 12)[None, :]
    ss = O.column_sq_norms(A)
    k = 5
    idx = O.topk_indices(ss, k)
    best = min(sum(ss[j] for j in range(12) if j not in c)
               for c in itertools.combinations(range(12), k))
    assert abs(sum(ss[np.setdiff1d(np.arange(12), idx)]) - best) <= 1e-12 * ss.sum()
    inp = W.tiny_fp32(0)
    A = O.decode(inp.A, "f32")
    ss = O.column_sq_norms(A)
    idx = O.topk_indices(ss, 128)
    mine = ss.sum() - ss[idx].sum()
    for t in range(100):
        r = np.random.default_rng(t).choice(256, 128, replace=False)
        assert mine <= ss.sum() - ss[r].sum()


# ------------------------------------------------------------------ planted mistakes

def _pins_hold(topk=None, reduced=None):
    """Run the identity/permutation/minimax pins against a (possibly mutated)
    top-k and reduced product; True when all hold."""
    topk = topk or O.topk_indices
    reduced = reduced or O.reduced_matmul
    try:
        rng = np.random.default_rng(7)
        A = rng.standard_normal((9, 12)) * np.arange(1, 13)[None, :]
        idx = topk(O.column_sq_norms(A), 6)
        Y = reduced(A, np.eye(12), idx)
        expect = np.zeros_like(A)
        expect[:, 6:] = A[:, 6:]
        if not np.array_equal(Y, expect):
            return False
        s = np.array([0.0, 5.0, 1.0, 5.0, 5.0, 2.0])
        if list(topk(s, 2)) != [1, 3]:
            return False
        rng = np.random.default_rng(8)
        A = rng.standard_normal((5, 10)) * (10 - np.arange(10))[None, :]
        p = rng.permutation(10)
        B = np.zeros((10, 10))
        B[np.arange(10), p] = 1.0
        idx = topk(O.column_sq_norms(A), 3)
        Y = reduced(A, B, idx)
        expect = np.zeros((5, 10))
        for j in [0, 1, 2]:
            expect[:, p[j]] = A[:, j]
        return np.array_equal(Y, expect)
    except Exception:
        return False


def test_pins_catch_planted_mistakes():
    assert _pins_hold()
    # smallest instead of largest scores
    assert not _pins_hold(topk=lambda s, k: np.sort(np.argsort(s, kind="stable")[:k]))
    # highest-index tie rule
    assert not _pins_hold(topk=lambda s, k: np.sort(
        (len(s) - 1 - np.lexsort((np.arange(len(s)), -s[::-1])))[:k]))
    # wrong operand: columns of B instead of rows
    assert not _pins_hold(reduced=lambda A, B, i: A[:, i] @ B[:, i].T)
    # dropped term: last kept index ignored
    assert not _pins_hold(reduced=lambda A, B, i: A[:, i[:-1]] @ B[i[:-1], :])
    # off-by-one in the gather
    assert not _pins_hold(reduced=lambda A, B, i: A[:, i] @ B[np.minimum(i + 1, B.shape[0] - 1), :])


# ------------------------------------------------------------------ int8 weight


def _w8_bruteforce(A, Bq, scale, rho):
    """Whole int8-weight path by enumeration and explicit loops: the k-subset
    with the largest sum of squared column norms (lowest indices first among
    equals), then Y[m][n] = sum over kept j of A[m][j] * Bq[j][n] * scale[n]."""
    M, d = A.shape
    N = Bq.shape[1]
    k = math.ceil(rho * d - 1e-9 * d)
    ss = [sum(A[m][j] ** 2 for m in range(M)) for j in range(d)]
    best = None
    for sub in itertools.combinations(range(d), k):
        key = (-sum(ss[j] for j in sub), sub)
        if best is None or key < best:
            best = key
    I = best[1]
    Y = [[0.0] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for j in I:
                acc += A[m][j] * float(Bq[j][n]) * float(scale[n])
            Y[m][n] = acc
    return np.array(Y), np.array(I)


@pytest.mark.parametrize("trial", range(4))
def test_w8_bruteforce_small(trial):
    rng = np.random.default_rng(100 + trial)
    M, d, N = 3, 8, 5
    A = rng.standard_normal((M, d)) * rng.uniform(0.2, 3.0, size=d)[None, :]
    Bq = rng.integers(-127, 128, size=(d, N)).astype(np.int8)
    scale = rng.uniform(1e-3, 5e-2, size=N).astype(np.float32)
    for rho in (0.25, 0.5, 0.75):
        Y, idx, _ = O.rmm_w8(A, Bq, scale, rho)
        Yb, Ib = _w8_bruteforce(A, Bq, scale, rho)
        np.testing.assert_array_equal(idx, Ib)
        np.testing.assert_allclose(Y, Yb, rtol=1e-12, atol=1e-15)


def test_w8_rho_one_factors_column_scale():
    """rho = 1: the product is the dense int8 product with column n scaled by
    scale[n] afterwards (distributivity; pins per-column, not per-row, scales)."""
    rng = np.random.default_rng(11)
    A = rng.standard_normal((6, 9))
    Bq = rng.integers(-127, 128, size=(9, 7)).astype(np.int8)
    scale = rng.uniform(0.5, 2.0, size=7).astype(np.float32)
    Y, idx, _ = O.rmm_w8(A, Bq, scale, 1.0)
    np.testing.assert_array_equal(idx, np.arange(9))
    dense_int = np.einsum("mj,jn->mn", A, Bq.astype(np.float64))
    np.testing.assert_allclose(Y, dense_int * scale.astype(np.float64)[None, :], rtol=1e-13, atol=1e-13)


def test_w8_unit_scale_is_plain_reduced_product():
    rng = np.random.default_rng(12)
    A = rng.standard_normal((4, 10)) * np.arange(1, 11)[None, :]
    Bq = rng.integers(-127, 128, size=(10, 3)).astype(np.int8)
    Y, idx, _ = O.rmm_w8(A, Bq, np.ones(3, np.float32), 0.4)
    Y2, idx2, _ = O.rmm(A, Bq.astype(np.float64), 0.4)
    np.testing.assert_array_equal(idx, idx2)
    np.testing.assert_array_equal(Y, Y2)


@pytest.mark.parametrize("rho", [0.3, 0.6])
def test_w8_error_bound(rho):
    """The error bound of the reduced product holds for the dequantised weight."""
    rng = np.random.default_rng(13)
    A = rng.standard_normal((16, 24)) * np.exp(rng.standard_normal(24))[None, :]
    Bq, scale = W.weight_int8(5, 24, 11)
    B = O.dequantize_w8(Bq, scale)
    Y, idx, _ = O.rmm_w8(A, Bq, scale, rho)
    rest = np.setdiff1d(np.arange(24), idx)
    err = np.linalg.norm(A @ B - Y)
    assert err <= np.linalg.norm(A[:, rest]) * np.linalg.norm(B[rest, :], 2) * (1 + 1e-9)


def test_weight_int8_is_absmax_storage():
    """Generated int8 weights use the full symmetric range per column."""
    q, s = W.weight_int8(3, 200, 33)
    assert q.dtype == np.int8 and s.dtype == np.float32
    assert np.all(np.abs(q.astype(np.int32)) <= 127)
    assert np.all(np.max(np.abs(q.astype(np.int32)), axis=0) == 127)
    assert np.all(s > 0)


def test_w8_pins_catch_planted_mistakes():
    """Each plausible mistake in the int8 product fails the brute-force pin."""
    rng = np.random.default_rng(200)
    M, d, N = 3, 8, 5
    A = rng.standard_normal((M, d)) * rng.uniform(0.2, 3.0, size=d)[None, :]
    Bq = rng.integers(-127, 128, size=(d, N)).astype(np.int8)
    scale = rng.uniform(1e-3, 5e-2, size=N).astype(np.float32)
    Yb, Ib = _w8_bruteforce(A, Bq, scale, 0.5)

    def holds(prod):
        Y = prod(A[:, Ib], Bq[Ib, :].astype(np.float64), scale.astype(np.float64))
        return np.allclose(Y, Yb, rtol=1e-12, atol=1e-15)

    assert holds(lambda a, q, s: a @ (q * s[None, :]))
    assert not holds(lambda a, q, s: a @ q)                                       # scale dropped
    assert not holds(lambda a, q, s: a @ (q * s[0]))                              # first column's scale for all
    assert not holds(lambda a, q, s: (a @ q) / s[None, :])                        # scale inverted
    assert not holds(lambda a, q, s: a @ (q * np.resize(s, q.shape[0])[:, None]))  # per-row scale
