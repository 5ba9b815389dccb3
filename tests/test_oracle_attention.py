"""Pins for the fp64 reduced-attention oracle: the dense special case against
torch's own causal attention (a library routine, fp64 on CPU), a closed-form
uniform-attention case, the grouped-query mapping, and the column-norm token
score against a library softmax.  CPU only."""
import math

import numpy as np
import pytest
import torch

from oracle import attention as OA
from oracle import rmm as O


def _rand(shape, seed, scale_per_dim=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape)
    if scale_per_dim:
        x *= np.exp(0.5 * rng.standard_normal(shape[-1]))[None, :]
    return x


def _sdpa(Q, K, V, scale=None):
    q, k, v = (torch.from_numpy(np.ascontiguousarray(t))[None, None] for t in (Q, K, V))
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale)
    return o[0, 0].numpy()


@pytest.mark.parametrize("S,D", [(64, 16), (97, 32), (128, 128)])
def test_dense_case_equals_library_attention(S, D):
    Q, K, V = (_rand((S, D), s) for s in (1, 2, 3))
    r = OA.attention_head(Q, K, V, 1.0, 1.0)
    np.testing.assert_array_equal(r["idx_d"], np.arange(D))
    np.testing.assert_array_equal(r["idx_t"], np.arange(S))
    ref = _sdpa(Q, K, V)
    assert np.max(np.abs(r["O"] - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_headdim_reduction_equals_library_on_kept_dims():
    S, D = 80, 32
    Q, K, V = (_rand((S, D), s) for s in (4, 5, 6))
    r = OA.attention_head(Q, K, V, 0.5, 1.0)
    ss = torch.from_numpy(Q).pow(2).sum(0)
    kept = np.sort(torch.topk(ss, 16).indices.numpy())
    np.testing.assert_array_equal(r["idx_d"], kept)
    # READING R2: original temperature 1/sqrt(D)
    ref = _sdpa(Q[:, kept], K[:, kept], V, scale=1.0 / math.sqrt(D))
    assert np.max(np.abs(r["O"] - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_uniform_attention_closed_form():
    """K = 0: every causal logit is 0, so P_ij = 1/(i+1) (j <= i),
    lse_i = log(i+1), t_j = sum_{i>=j} 1/(i+1)^2 (strictly decreasing in j, so
    the kept tokens are the first k_t), O_i = sum_{j<=min(i,k_t-1)} V_j/(i+1)."""
    S, D = 50, 8
    Q = _rand((S, D), 7)
    K = np.zeros((S, D))
    V = _rand((S, D), 8)
    r = OA.attention_head(Q, K, V, 0.5, 0.3)
    kt = O.k_from_rho(0.3, S)
    i = np.arange(S)
    np.testing.assert_allclose(r["lse"], np.log(i + 1.0), rtol=0, atol=1e-14)
    t = np.array([sum(1.0 / (ii + 1) ** 2 for ii in range(j, S)) for j in range(S)])
    np.testing.assert_allclose(r["t"], t, rtol=1e-13)
    np.testing.assert_array_equal(r["idx_t"], np.arange(kt))
    O_ref = np.array([V[:min(ii, kt - 1) + 1].sum(0) / (ii + 1) for ii in range(S)])
    np.testing.assert_allclose(r["O"], O_ref, rtol=1e-12, atol=1e-14)


def test_token_scores_are_column_norms_of_library_softmax():
    S, D = 70, 16
    Q, K, V = (_rand((S, D), s) for s in (9, 10, 11))
    r = OA.attention_head(Q, K, V, 0.75, 0.5)
    kd = r["idx_d"]
    logits = torch.from_numpy(Q[:, kd] @ K[:, kd].T / math.sqrt(D))
    logits = logits.masked_fill(~torch.tril(torch.ones(S, S, dtype=torch.bool)), float("-inf"))
    P = torch.softmax(logits, dim=-1).numpy()
    np.testing.assert_allclose(r["t"], (P ** 2).sum(0), rtol=1e-12)
    np.testing.assert_allclose(r["lse"], torch.logsumexp(logits, -1).numpy(), rtol=1e-13)
    # READING R5: P not renormalised over the kept tokens
    it = r["idx_t"]
    np.testing.assert_allclose(r["O"], P[:, it] @ V[it], rtol=1e-12, atol=1e-14)
    # a query whose causal window holds no kept token gets a zero row
    first = it.min()
    assert np.all(r["O"][:first] == 0.0)


def test_gqa_mapping_equals_repeated_kv():
    rng = np.random.default_rng(12)
    B, Hq, Hkv, S, D = 2, 4, 2, 40, 16
    Q = rng.standard_normal((B, Hq, S, D))
    K = rng.standard_normal((B, Hkv, S, D))
    V = rng.standard_normal((B, Hkv, S, D))
    g = OA.reduced_attention(Q, K, V, 0.5, 0.5)
    m = OA.reduced_attention(Q, np.repeat(K, 2, axis=1), np.repeat(V, 2, axis=1), 0.5, 0.5)
    for key in g:
        np.testing.assert_array_equal(g[key], m[key])
    assert [OA.kv_head_of(h, 32, 8) for h in (0, 3, 4, 31)] == [0, 0, 1, 7]


def test_planted_mistake_renormalised_pv_is_caught():
    """A renormalising variant (not READING R5) fails the closed-form pin."""
    S, D = 50, 8
    Q = _rand((S, D), 7)
    V = _rand((S, D), 8)
    r = OA.attention_head(Q, np.zeros((S, D)), V, 0.5, 0.3)
    kt = O.k_from_rho(0.3, S)
    renorm = np.array([V[:min(ii, kt - 1) + 1].mean(0) for ii in range(S)])
    assert not np.allclose(r["O"], renorm)


def test_restricted_forms_agree_with_full_head():
    S, D = 90, 16
    Q, K, V = (_rand((S, D), s) for s in (13, 14, 15))
    r = OA.attention_head(Q, K, V, 0.5, 0.4)
    idx_d = OA.head_dim_selection(Q, 0.5)
    np.testing.assert_array_equal(idx_d, r["idx_d"])
    rows = np.arange(S)
    lse = OA.lse_rows(Q, K, idx_d, rows)
    np.testing.assert_allclose(lse, r["lse"], rtol=1e-13, atol=1e-13)
    t = OA.token_scores(Q, K, idx_d, lse, np.arange(S))
    np.testing.assert_allclose(t, r["t"], rtol=1e-12)
    some = np.array([0, 7, 44, 89])
    O = OA.out_rows(Q, K, V, idx_d, lse[some], r["idx_t"], some)
    np.testing.assert_allclose(O, r["O"][some], rtol=1e-12, atol=1e-14)


def test_restricted_forms_uniform_closed_form():
    S, D = 40, 8
    Q = _rand((S, D), 16)
    K = np.zeros((S, D))
    V = _rand((S, D), 17)
    idx_d = OA.head_dim_selection(Q, 1.0)
    lse = OA.lse_rows(Q, K, idx_d, np.arange(S))
    np.testing.assert_allclose(lse, np.log(np.arange(1, S + 1)), atol=1e-14)
    t = OA.token_scores(Q, K, idx_d, lse, [0, 5, S - 1])
    ref = [sum(1.0 / (i + 1) ** 2 for i in range(j, S)) for j in (0, 5, S - 1)]
    np.testing.assert_allclose(t, ref, rtol=1e-13)
    O = OA.out_rows(Q, K, V, idx_d, lse[[3, 20]], [0, 2, 30], [3, 20])
    np.testing.assert_allclose(O, [(V[0] + V[2]) / 4, (V[0] + V[2]) / 21], rtol=1e-13)
