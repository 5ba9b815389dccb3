"""Pins of the block-driver oracle: bf16 rounding against torch's conversion,
SiLU at known points, brute force over every subset on a tiny MLP block, the
dense special case against torch's fp64 MLP, and planted mistakes."""
import itertools
import math

import numpy as np
import pytest
import torch

from oracle import block as OB
from oracle import rmm as O


def test_round_bf16_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(5000) * 10.0 ** rng.uniform(-3, 3, 5000),
                        [1.0, -1.0, 0.73105857863, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -9, 3.0 * 2.0 ** -9 + 1.0]])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(OB.round_bf16(x), ref)


def test_silu_known_values():
    G = np.array([0.0, 1.0, -1.0, 30.0, -30.0])
    U = np.ones(5)
    H = OB.silu_mul_bf16(G, U)
    assert H[0] == 0.0
    assert H[1] == 187.0 / 256.0            # 1 / (1 + e^-1) = 0.7310... -> 0.73046875 in bf16
    assert H[2] == -69.0 / 256.0            # -1 / (1 + e) = -0.2689... -> -0.26953125
    assert H[3] == 30.0
    assert abs(H[4]) < 1e-11


def _brute_block(X, Wu, Wg, Wd, rho_up, rho_down):
    """The block by enumeration and loops: subsets maximising the summed column
    scores (lowest indices among equals), products by explicit sums, bf16
    rounding through torch."""
    def best(scores, k):
        top = None
        for sub in itertools.combinations(range(len(scores)), k):
            key = (-sum(scores[i] for i in sub), sub)
            if top is None or key < top:
                top = key
        return list(top[1])

    def bf16(v):
        return float(torch.tensor(v, dtype=torch.float64).to(torch.bfloat16).to(torch.float64))

    M, dm = X.shape
    dff = Wu.shape[1]
    I = best([sum(X[m][j] ** 2 for m in range(M)) for j in range(dm)], math.ceil(rho_up * dm - 1e-9 * dm))
    U = [[bf16(sum(X[m][j] * Wu[j][n] for j in I)) for n in range(dff)] for m in range(M)]
    G = [[bf16(sum(X[m][j] * Wg[j][n] for j in I)) for n in range(dff)] for m in range(M)]
    H = [[bf16(G[m][n] / (1.0 + math.exp(-G[m][n])) * U[m][n]) for n in range(dff)] for m in range(M)]
    J = best([sum(H[m][n] ** 2 for m in range(M)) for n in range(dff)], math.ceil(rho_down * dff - 1e-9 * dff))
    Y = [[sum(H[m][n] * Wd[n][c] for n in J) for c in range(dm)] for m in range(M)]
    return np.array(Y), I, J


@pytest.mark.parametrize("seed", range(3))
def test_mlp_block_bruteforce(seed):
    rng = np.random.default_rng(10 + seed)
    M, dm, dff = 3, 6, 8
    X = rng.standard_normal((M, dm)) * rng.uniform(0.3, 3.0, dm)
    Wu, Wg = rng.standard_normal((dm, dff)), rng.standard_normal((dm, dff))
    Wd = rng.standard_normal((dff, dm))
    r = OB.mlp_block(X, Wu, Wg, Wd, 0.5, 0.5)
    Y, I, J = _brute_block(X, Wu, Wg, Wd, 0.5, 0.5)
    np.testing.assert_array_equal(r["I"], I)
    np.testing.assert_array_equal(r["J"], J)
    np.testing.assert_allclose(r["Y"], Y, rtol=1e-12, atol=1e-12)


def test_mlp_block_dense_special_case():
    """rho = 1 everywhere: the dense gated MLP with bf16 intermediates, from
    torch's fp64 silu and matmul."""
    rng = np.random.default_rng(4)
    X = rng.standard_normal((5, 16))
    Wu, Wg, Wd = rng.standard_normal((16, 24)), rng.standard_normal((16, 24)), rng.standard_normal((24, 16))
    r = OB.mlp_block(X, Wu, Wg, Wd, 1.0, 1.0)
    t = lambda a: torch.from_numpy(a)
    b = lambda z: z.to(torch.bfloat16).to(torch.float64)
    U, G = b(t(X) @ t(Wu)), b(t(X) @ t(Wg))
    H = b(torch.nn.functional.silu(G) * U)
    np.testing.assert_allclose(r["H"], H.numpy(), rtol=0, atol=0)
    np.testing.assert_allclose(r["Y"], (H @ t(Wd)).numpy(), rtol=1e-12, atol=1e-12)


def test_matmul_shared_is_one_selection():
    """Every product uses the index set of A alone: against the single-product
    path on each weight."""
    rng = np.random.default_rng(5)
    A = rng.standard_normal((7, 20)) * np.arange(1, 21)
    Bs = [rng.standard_normal((20, n)) for n in (3, 9, 4)]
    Ys, I, _ = OB.matmul_shared(A, Bs, 0.35)
    for B, Y in zip(Bs, Ys):
        Yr, Ir, _ = O.rmm(A, B, 0.35)
        np.testing.assert_array_equal(I, Ir)
        np.testing.assert_array_equal(Y, Yr)
    np.testing.assert_array_equal(I, np.arange(13, 20))    # column scale grows with the index


def test_block_pins_catch_planted_mistakes(monkeypatch):
    rng = np.random.default_rng(11)
    M, dm, dff = 3, 6, 8
    X = rng.standard_normal((M, dm)) * rng.uniform(0.3, 3.0, dm)
    Wu, Wg = rng.standard_normal((dm, dff)), rng.standard_normal((dm, dff))
    Wd = rng.standard_normal((dff, dm))
    Yb, I, J = _brute_block(X, Wu, Wg, Wd, 0.5, 0.5)

    def holds():
        r = OB.mlp_block(X, Wu, Wg, Wd, 0.5, 0.5)
        return (np.array_equal(r["I"], I) and np.array_equal(r["J"], J)
                and np.allclose(r["Y"], Yb, rtol=1e-12, atol=1e-12))
    assert holds()
    real_silu, real_round = OB.silu_mul_bf16, OB.round_bf16
    # gate and up swapped
    monkeypatch.setattr(OB, "silu_mul_bf16", lambda G, U: real_silu(U, G))
    assert not holds()
    # sigmoid instead of SiLU
    monkeypatch.setattr(OB, "silu_mul_bf16", lambda G, U: real_round(U / (1.0 + np.exp(-np.asarray(G)))))
    assert not holds()
    monkeypatch.setattr(OB, "silu_mul_bf16", real_silu)
    # no bf16 storage of the intermediates
    monkeypatch.setattr(OB, "round_bf16", lambda x: np.asarray(x, dtype=np.float64))
    assert not holds()
    monkeypatch.setattr(OB, "round_bf16", real_round)
    # down projection scored on the activation before the gate
    real_css = OB.column_sq_norms
    calls = []

    def css(A):
        calls.append(1)
        return real_css(A) if len(calls) == 1 else real_css(np.ones_like(A))
    monkeypatch.setattr(OB, "column_sq_norms", css)
    assert not holds()
    monkeypatch.setattr(OB, "column_sq_norms", real_css)
    assert holds()
