"""GPU parity of reduced attention (rmm_attention) against the fp64 oracle.

Inputs are the seeded attention workload; kv-groups are redrawn (the
generator's `attempt`) until every q-head's head_dim boundary has a relative
score gap >= 2e-5 and its token boundary a relative gap >= 1e-3, so the fp32
GPU ranking and the fp64 oracle ranking must agree and index sets are compared
bit-exactly.  At full size, where such margins cannot be drawn in reasonable
time, the token set is checked for validity instead (every kept score at
least, every dropped score at most, the k-th largest oracle score within
1e-4) and O is compared against the oracle evaluated on the GPU's set.

Tolerances, from the arithmetic: logits are exact bf16 products summed in
fp32; lse to 2e-5 absolute; token scores to 1e-4 relative; O elementwise
within 2^-8 * sum_j P_ij |V_j| (P is rounded to bf16 before the PV product)
plus the fp32 summation bound and, for bf16 output, one bf16 ulp; relative
Frobenius of O <= 5e-3."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from oracle import attention as OA
from oracle.conditioning import boundary_gaps
from tests.helpers import bf16_tensor, bf16_ulp, rel_fro, to_f64

pytestmark = pytest.mark.gpu
R = None


@pytest.fixture(scope="module", autouse=True)
def lib():
    global R
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import input_adaptive_reduced_score_b200 as mod
    R = mod
    R.rmm_device_error(clear=True)
    yield mod
    assert R.rmm_device_error(clear=True) == 0


def draw(B, Hq, Hkv, S, D, rho_d, rho_t, seed=3, max_attempts=60):
    """Attention inputs whose every q-head has clear selection margins."""
    G = Hq // Hkv
    kd, kt = oracle.k_from_rho(rho_d, D), oracle.k_from_rho(rho_t, S)
    attempts = [0] * Hkv
    for g in range(Hkv):
        while True:
            inp = W.attention(seed, B, Hq, Hkv, S, D, rho_d, rho_t, attempts)
            Q, K, V = (oracle.decode(x, "bf16") for x in (inp.Q, inp.K, inp.V))
            good = True
            for b in range(B):
                for h in range(g * G, (g + 1) * G):
                    if kd < D:
                        gd, _ = boundary_gaps(oracle.column_sq_norms(Q[b, h]), [kd])
                        good &= gd[kd] >= 2e-5
                    if kt < S and good:
                        r = OA.attention_head(Q[b, h], K[b, g], V[b, g], rho_d, rho_t)
                        gt, _ = boundary_gaps(r["t"], [kt])
                        good &= gt[kt] >= 1e-3
            if good:
                break
            attempts[g] += 1
            assert attempts[g] < max_attempts, "could not draw clear margins"
    return W.attention(seed, B, Hq, Hkv, S, D, rho_d, rho_t, attempts)


def run_gpu(inp, out_dtype=torch.float32):
    B, Hq, Hkv, S, D = inp.shape
    Qt, Kt, Vt = (bf16_tensor(x) for x in (inp.Q, inp.K, inp.V))
    kd, kt = oracle.k_from_rho(inp.rho_d, D), oracle.k_from_rho(inp.rho_t, S)
    idx_d = torch.full((B * Hq, kd), -1, dtype=torch.int32, device="cuda")
    idx_t = torch.full((B * Hq, kt), -1, dtype=torch.int32, device="cuda")
    lse = torch.empty((B * Hq, S), dtype=torch.float32, device="cuda")
    tsc = torch.empty((B * Hq, S), dtype=torch.float32, device="cuda")
    O = R.rmm_attention(Qt, Kt, Vt, inp.rho_d, inp.rho_t, out_dtype=out_dtype, idx_d=idx_d, idx_t=idx_t,
                        lse=lse, tscore=tsc)
    assert R.rmm_device_error(clear=True) == 0
    return (to_f64(O), idx_d.cpu().numpy().reshape(B, Hq, kd), idx_t.cpu().numpy().reshape(B, Hq, kt),
            lse.cpu().numpy().reshape(B, Hq, S), tsc.cpu().numpy().reshape(B, Hq, S))


def check_o(got, ref, P, V, idx_t, kt, bf16_out):
    _bound_check(got, ref, np.abs(P[:, idx_t]) @ np.abs(V[idx_t]), kt, bf16_out)


CASES = [  # B, Hq, Hkv, S, D, rho_d, rho_t
    (1, 2, 2, 128, 128, 0.5, 0.5),
    (1, 4, 2, 256, 128, 0.5, 0.5),     # GQA
    (2, 2, 1, 300, 64, 0.5, 0.5),      # ragged S, D = 64
    (1, 2, 2, 384, 128, 1.0, 1.0),     # dense special case
    (1, 2, 2, 200, 128, 0.75, 0.3),
    (1, 2, 2, 130, 64, 1.0, 0.5),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}Hq{}Hkv{}S{}D{}rd{}rt{}".format(*c))
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_attention_parity(case, out_dtype):
    B, Hq, Hkv, S, D, rho_d, rho_t = case
    inp = draw(B, Hq, Hkv, S, D, rho_d, rho_t)
    O, idx_d, idx_t, lse, tsc = run_gpu(inp, out_dtype)
    Q, K, V = (oracle.decode(x, "bf16") for x in (inp.Q, inp.K, inp.V))
    kt = oracle.k_from_rho(rho_t, S)
    errs = []
    for b in range(B):
        for h in range(Hq):
            g = OA.kv_head_of(h, Hq, Hkv)
            r = OA.attention_head(Q[b, h], K[b, g], V[b, g], rho_d, rho_t, return_p=True)
            np.testing.assert_array_equal(idx_d[b, h], r["idx_d"])
            np.testing.assert_allclose(lse[b, h], r["lse"], rtol=0, atol=2e-5)
            np.testing.assert_allclose(tsc[b, h], r["t"], rtol=1e-4, atol=0)
            np.testing.assert_array_equal(idx_t[b, h], r["idx_t"])
            check_o(O[b, h], r["O"], r["P"], V[b, g], r["idx_t"], kt, out_dtype == torch.bfloat16)
            errs.append(rel_fro(O[b, h], r["O"]))
    assert max(errs) <= 5e-3, errs


def test_attention_rows_without_kept_tokens_are_zero():
    """Two 'sink' keys (5 and 9) that every query attends to carry the largest
    token scores; with k_t = 2 only they are kept, so queries 0..4 have no kept
    token in their causal window and their output rows are exactly zero."""
    S, D = 256, 64
    rng = np.random.default_rng(21)
    c = np.linspace(0.5, 1.5, D)
    Qf = c[None, :] + 0.05 * rng.standard_normal((S, D))
    Kf = 0.05 * rng.standard_normal((S, D))
    Kf[[5, 9]] = 0.9 * c[None, :]
    Vf = rng.standard_normal((S, D))
    enc = lambda x: W.f32_to_bf16_bits(x).reshape(1, 1, S, D)
    inp = W.AttentionInputs("sinks", enc(Qf), enc(Kf), enc(Vf), 1.0, 2.0 / S, 0)
    O, _, idx_t, _, _ = run_gpu(inp)
    np.testing.assert_array_equal(idx_t[0, 0], [5, 9])
    assert np.all(O[0, 0, :5] == 0.0) and np.all(np.abs(O[0, 0, 5:]).sum(1) > 0)
    Q, K, V = (oracle.decode(x[0, 0], "bf16") for x in (inp.Q, inp.K, inp.V))
    r = OA.attention_head(Q, K, V, 1.0, 2.0 / S, return_p=True)
    np.testing.assert_array_equal(r["idx_t"], [5, 9])
    check_o(O[0, 0], r["O"], r["P"], V, r["idx_t"], 2, False)


def _bound_check(got, ref, absterm, kt, bf16_out):
    bound = (2.0 ** -8 + 2e-5 + kt * 2.0 ** -24) * absterm + 1e-30
    if bf16_out:
        bound = bound + bf16_ulp(np.maximum(np.abs(got), np.abs(ref)))
    bad = np.abs(got - ref) > bound
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside the bound"


@pytest.mark.slow
@pytest.mark.parametrize("S,Hq,Hkv,seed,heads", [(8192, 32, 32, 3, [0, 31]), (32768, 32, 8, 4, [13])])
def test_attention_full_size_sampled_heads(S, Hq, Hkv, seed, heads):
    """Full-size workloads (32 heads at 8192 tokens; GQA 32/8 at 32768 tokens),
    bf16 output: every head runs on the GPU; sampled heads are checked with the
    oracle's row/column-restricted forms: the head_dim set (bit-exact where its
    margin is clear), lse of every row, token scores of every column, validity
    of the kept token set, and O on 256 sampled rows given that set."""
    inp = W.attention(seed, 1, Hq, Hkv, S, 128, 0.5, 0.5)
    O, idx_d, idx_t, lse, tsc = run_gpu(inp, torch.bfloat16)
    kd, kt = 64, oracle.k_from_rho(0.5, S)
    rng = np.random.default_rng(S)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, S - 1], rng.integers(0, S, 251)]))
    for h in heads:
        g = OA.kv_head_of(h, Hq, Hkv)
        Q, K, V = (oracle.decode(x, "bf16") for x in (inp.Q[0, h], inp.K[0, g], inp.V[0, g]))
        ssq = oracle.column_sq_norms(Q)
        gd, _ = boundary_gaps(ssq, [kd])
        if gd[kd] >= 2e-5:
            np.testing.assert_array_equal(idx_d[0, h], OA.head_dim_selection(Q, 0.5))
        else:  # a valid top-k within fp32 scoring error
            T = np.sort(ssq)[::-1][kd - 1]
            m = np.zeros(128, bool)
            m[idx_d[0, h]] = True
            assert ssq[m].min() >= T * (1 - 1e-5) and ssq[~m].max() <= T * (1 + 1e-5)
        sel = idx_d[0, h]
        L = OA.lse_rows(Q, K, sel, np.arange(S))
        np.testing.assert_allclose(lse[0, h], L, rtol=0, atol=5e-5)
        t = OA.token_scores(Q, K, sel, L, np.arange(S))
        np.testing.assert_allclose(tsc[0, h], t, rtol=2e-4, atol=0)
        T = np.sort(t)[::-1][kt - 1]
        kept = np.zeros(S, bool)
        kept[idx_t[0, h]] = True
        assert kept.sum() == kt and np.all(np.diff(idx_t[0, h]) > 0)
        assert t[kept].min() >= T * (1 - 2e-4) and t[~kept].max() <= T * (1 + 2e-4)
        ref = OA.out_rows(Q, K, V, sel, L[rows], idx_t[0, h], rows)
        absterm = OA.out_rows(Q, K, np.abs(V), sel, L[rows], idx_t[0, h], rows)
        _bound_check(O[0, h][rows], ref, absterm, kt, True)
        assert rel_fro(O[0, h][rows], ref) <= 5e-3
