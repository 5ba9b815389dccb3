"""Pins of the decode-attention oracle (one query token over a KV cache) to
facts outside itself: the dense special case against torch's fp64 attention,
brute force over every head_dim and token subset on tiny inputs, a closed
form for identical keys, the grouped-query head mapping, and planted
mistakes that each pin must catch."""
import itertools
import math

import numpy as np
import pytest
import torch

from oracle import decode_attention as OD


def _bruteforce(q, K, V, rho_d, rho_t):
    """Everything by enumeration and explicit loops, from the readings: the
    head_dim subset with the largest sum of q_c^2 (lowest indices among
    equals), logits with scale 1/sqrt(D), the softmax, the token subset with
    the largest sum of P_j^2 (lowest indices among equals), O = sum P_j V_j."""
    L, D = K.shape
    kd = math.ceil(rho_d * D - 1e-9 * D)
    kt = math.ceil(rho_t * L - 1e-9 * L)

    def best(values, k):
        top = None
        for sub in itertools.combinations(range(len(values)), k):
            key = (-sum(values[i] for i in sub), sub)
            if top is None or key < top:
                top = key
        return list(top[1])

    Id = best([q[c] * q[c] for c in range(D)], kd)
    logits = [sum(q[c] * K[j][c] for c in Id) / math.sqrt(D) for j in range(L)]
    m = max(logits)
    z = sum(math.exp(x - m) for x in logits)
    P = [math.exp(x - m) / z for x in logits]
    It = best([p * p for p in P], kt)
    O = [sum(P[j] * V[j][c] for j in It) for c in range(V.shape[1])]
    return np.array(O), np.array(Id), np.array(It), m + math.log(z)


def _tiny(seed):
    rng = np.random.default_rng(seed)
    L, D = 7, 4
    q = rng.standard_normal(D) * rng.uniform(0.3, 2.0, D)
    K = rng.standard_normal((L, D))
    V = rng.standard_normal((L, 3))
    return q, K, V


@pytest.mark.parametrize("seed", range(5))
@pytest.mark.parametrize("rho_d,rho_t", [(0.5, 0.4), (0.75, 0.6), (0.25, 0.3)])
def test_decode_bruteforce(seed, rho_d, rho_t):
    q, K, V = _tiny(seed)
    r = OD.decode_attention_head(q, K, V, rho_d, rho_t)
    O, Id, It, lse = _bruteforce(q, K, V, rho_d, rho_t)
    np.testing.assert_array_equal(r["idx_d"], Id)
    np.testing.assert_array_equal(r["idx_t"], It)
    np.testing.assert_allclose(r["O"], O, rtol=1e-12, atol=1e-14)
    assert abs(r["lse"] - lse) < 1e-12


def test_decode_dense_is_softmax_attention():
    """rho_d = rho_t = 1: textbook attention of one query, from torch's fp64 SDPA."""
    rng = np.random.default_rng(3)
    L, D = 50, 16
    q, K, V = rng.standard_normal(D), rng.standard_normal((L, D)), rng.standard_normal((L, D))
    r = OD.decode_attention_head(q, K, V, 1.0, 1.0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None, None, :], torch.from_numpy(K)[None, None], torch.from_numpy(V)[None, None])
    np.testing.assert_allclose(r["O"], ref[0, 0, 0].numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(r["lse"], torch.logsumexp(torch.from_numpy(K @ q) / math.sqrt(D), 0).item(),
                               rtol=1e-13)


def test_decode_identical_keys_closed_form():
    """All keys equal: P is uniform 1/L, every token ties, the lowest k_t are kept,
    O = (1/L) * sum of the first k_t values (not their mean: no renormalisation)."""
    rng = np.random.default_rng(4)
    L, D = 20, 8
    q = rng.standard_normal(D)
    K = np.tile(rng.standard_normal(D), (L, 1))
    V = rng.standard_normal((L, D))
    r = OD.decode_attention_head(q, K, V, 0.5, 0.3)
    kt = 6
    np.testing.assert_array_equal(r["idx_t"], np.arange(kt))
    np.testing.assert_allclose(r["O"], V[:kt].sum(0) / L, rtol=1e-13)


def test_decode_gqa_mapping_and_cache_length():
    """q-head h reads kv-head h * Hkv / Hq; only the first L cache rows count."""
    rng = np.random.default_rng(5)
    B, Hq, Hkv, Lmax, L, D = 2, 4, 2, 12, 9, 8
    q = rng.standard_normal((B, Hq, D))
    K = rng.standard_normal((B, Hkv, Lmax, D))
    V = rng.standard_normal((B, Hkv, Lmax, D))
    out = OD.decode_attention(q, K, V, L, 0.5, 0.5)
    for b in range(B):
        for h in range(Hq):
            r = OD.decode_attention_head(q[b, h], K[b, h // 2, :L], V[b, h // 2, :L], 0.5, 0.5)
            np.testing.assert_array_equal(out["O"][b, h], r["O"])
            np.testing.assert_array_equal(out["idx_t"][b, h], r["idx_t"])


def _pins_hold():
    try:
        for seed in range(3):
            q, K, V = _tiny(seed)
            r = OD.decode_attention_head(q, K, V, 0.5, 0.4)
            O, Id, It, _ = _bruteforce(q, K, V, 0.5, 0.4)
            if not (np.array_equal(r["idx_d"], Id) and np.array_equal(r["idx_t"], It)
                    and np.allclose(r["O"], O, rtol=1e-12, atol=1e-14)):
                return False
        test_decode_identical_keys_closed_form()
        return True
    except (AssertionError, ValueError, IndexError):
        return False


def test_decode_pins_catch_planted_mistakes(monkeypatch):
    assert _pins_hold()
    real_topk, real_k = OD.topk_indices, OD.k_from_rho
    # smallest instead of largest scores
    monkeypatch.setattr(OD, "topk_indices", lambda s, k: np.sort(np.argsort(np.asarray(s), kind="stable")[:k]))
    assert not _pins_hold()
    monkeypatch.setattr(OD, "topk_indices", real_topk)
    # k from floor instead of ceil
    monkeypatch.setattr(OD, "k_from_rho", lambda rho, d: max(1, int(math.floor(rho * d))))
    assert not _pins_hold()
    monkeypatch.setattr(OD, "k_from_rho", real_k)
    # P renormalised over the kept tokens
    real_head = OD.decode_attention_head

    def renorm(q, K, V, rho_d, rho_t, scale=None):
        r = real_head(q, K, V, rho_d, rho_t, scale)
        P = np.exp(r["logits"] - r["lse"])
        r["O"] = r["O"] / P[r["idx_t"]].sum()
        return r
    monkeypatch.setattr(OD, "decode_attention_head", renorm)
    assert not _pins_hold()
    # temperature of the reduced head_dim instead of the full one
    monkeypatch.setattr(OD, "decode_attention_head",
                        lambda q, K, V, rd, rt, scale=None: real_head(q, K, V, rd, rt,
                                                                     1.0 / math.sqrt(OD.k_from_rho(rd, K.shape[1]))))
    assert not _pins_hold()
    monkeypatch.setattr(OD, "decode_attention_head", real_head)
    assert _pins_hold()
