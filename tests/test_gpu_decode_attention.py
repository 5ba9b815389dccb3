"""GPU parity of reduced decode attention (rmm_decode_attention) against the
fp64 oracle: one new query token per sequence over a KV cache.

Inputs are the seeded decode workload; a kv-group is redrawn (the generator's
`attempt`) until every q-head's token boundary has a logit gap >= 1e-4
between the k_t-th and (k_t+1)-th largest logits (the fp32 logits are within
about 2e-5 of the fp64 ones), so index sets are compared bit-exactly.  At
the benchmarked size and on the longest rows no redraw is made: there the
token set must be the exact top-k of the GPU's own logits, and O is checked
against the oracle's P over that set.  The head_dim selection needs no
margin: it ranks |q_c|, exactly the order of q_c^2.
Unused cache capacity holds 1e4, so a read past L would show.

Tolerances, from the arithmetic: logits are sums of exact bf16 products in
fp32 (at most 2^-24 per term of sum |q K| times the scale, plus the scale's
rounding); lse to 2e-5 absolute; O elementwise within
(k_t 2^-24 + 1e-5) * sum_{j in I_t} P_j |V_j| (fp32 sum; P from the fast
exponential of an fp32 logit) plus one bf16 ulp for bf16 output."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from oracle import decode_attention as OD
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


def _token_gap(logits, kt):
    if kt >= len(logits):
        return math.inf
    s = np.sort(logits)[::-1]
    return s[kt - 1] - s[kt]


def draw(B, Hq, Hkv, L, Lmax, D, rho_d, rho_t, seed=5, max_attempts=60):
    G = Hq // Hkv
    kt = oracle.k_from_rho(rho_t, L)
    attempts = [0] * Hkv
    for g in range(Hkv):
        while True:
            inp = W.decode_attention(seed, B, Hq, Hkv, L, D, rho_d, rho_t, Lmax, attempts)
            q, K, V = (oracle.decode(x, "bf16") for x in (inp.q, inp.K, inp.V))
            heads = [(b, h) for b in range(B) for h in range(g * G, (g + 1) * G)]
            r = OD.decode_attention(q, K, V, L, rho_d, rho_t, heads=heads)
            if all(_token_gap(r["logits"][b, h], kt) >= 1e-4 for b, h in heads):
                break
            attempts[g] += 1
            assert attempts[g] < max_attempts, "could not draw clear margins"
    return W.decode_attention(seed, B, Hq, Hkv, L, D, rho_d, rho_t, Lmax, attempts)


CASES = [  # B, Hq, Hkv, L, Lmax, D, rho_d, rho_t
    (1, 2, 2, 300, 300, 128, 0.5, 0.5),
    (2, 8, 2, 1000, 1024, 128, 0.5, 0.5),     # grouped query heads, cache capacity above L
    (1, 4, 1, 777, 800, 64, 0.5, 0.3),        # D = 64
    (1, 16, 1, 257, 257, 128, 0.75, 0.6),     # 16 q-heads per kv-head; one token past a chunk
    (3, 2, 2, 1, 4, 128, 0.5, 0.5),           # a single cached token
    (1, 2, 2, 2048, 2048, 128, 1.0, 1.0),     # dense special case
    (1, 4, 4, 5000, 5000, 128, 0.5, 0.5),     # token top-k on one 1024-thread CTA per head
    (1, 2, 2, 60000, 60000, 128, 0.5, 0.5),   # token top-k on clusters of 8 CTAs, a short last slice
    (4, 4, 4, 20000, 20000, 128, 0.5, 0.5),   # clusters of 4 CTAs, 16 rows
    (10, 8, 8, 3000, 3000, 128, 0.5, 0.5),    # 80 rows
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}Hq{}Hkv{}L{}Lmax{}D{}rd{}rt{}".format(*c))
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_decode_attention_parity(case, out_dtype):
    B, Hq, Hkv, L, Lmax, D, rho_d, rho_t = case
    inp = draw(B, Hq, Hkv, L, Lmax, D, rho_d, rho_t)
    q, K, V = (oracle.decode(x, "bf16") for x in (inp.q, inp.K, inp.V))
    ref = OD.decode_attention(q, K, V, L, rho_d, rho_t)
    kd, kt = oracle.k_from_rho(rho_d, D), oracle.k_from_rho(rho_t, L)
    idx_d = torch.full((B * Hq, kd), -1, dtype=torch.int32, device="cuda")
    idx_t = torch.full((B * Hq, kt), -1, dtype=torch.int32, device="cuda")
    lse = torch.empty(B * Hq, dtype=torch.float32, device="cuda")
    logits = torch.empty((B * Hq, L), dtype=torch.float32, device="cuda")
    O = R.rmm_decode_attention(bf16_tensor(inp.q), bf16_tensor(inp.K), bf16_tensor(inp.V), L, rho_d, rho_t,
                               out_dtype=out_dtype, idx_d=idx_d, idx_t=idx_t, lse=lse, logits=logits)
    assert R.rmm_device_error(clear=True) == 0
    np.testing.assert_array_equal(idx_d.cpu().numpy().reshape(B, Hq, kd), ref["idx_d"])
    np.testing.assert_array_equal(idx_t.cpu().numpy().reshape(B, Hq, kt), ref["idx_t"])
    scale = 1.0 / math.sqrt(D)
    got_s = logits.cpu().numpy().astype(np.float64).reshape(B, Hq, L)
    got_o = to_f64(O)
    for b in range(B):
        for h in range(Hq):
            g = h * Hkv // Hq
            Id = ref["idx_d"][b, h]
            absdot = scale * (np.abs(K[b, g, :L][:, Id]) @ np.abs(q[b, h, Id]))
            assert np.all(np.abs(got_s[b, h] - ref["logits"][b, h]) <= D * 2.0 ** -24 * absdot * 1.01 + 1e-6)
            It = ref["idx_t"][b, h]
            P = np.exp(ref["logits"][b, h] - ref["lse"][b, h])
            absw = P[It] @ np.abs(V[b, g, It])
            bound = (kt * 2.0 ** -24 + 1e-5) * absw + 1e-30
            if out_dtype == torch.bfloat16:
                bound = bound + bf16_ulp(np.maximum(np.abs(got_o[b, h]), np.abs(ref["O"][b, h])))
            assert np.all(np.abs(got_o[b, h] - ref["O"][b, h]) <= bound), (b, h)
    np.testing.assert_allclose(lse.cpu().numpy().astype(np.float64).reshape(B, Hq), ref["lse"], rtol=0, atol=2e-5)
    assert rel_fro(got_o, ref["O"]) <= (2e-3 if out_dtype == torch.bfloat16 else 1e-5)
    # without the optional outputs the token top-k writes only its bitmap:
    # the same kept set, so the same bits of O
    O2 = R.rmm_decode_attention(bf16_tensor(inp.q), bf16_tensor(inp.K), bf16_tensor(inp.V), L, rho_d, rho_t,
                                out_dtype=out_dtype)
    assert torch.equal(O2, O)


def _check_own_selection(inp, B, Hq, Hkv, L, D, rho_d, rho_t, heads):
    """Parity where the token boundary is not drawn clear: idx_d, the logits
    and lse against the oracle; idx_t must be the exact top-k (lowest index
    on ties) of the GPU's own fp32 logits; O against the reduced PV product of
    the oracle's P over that index set, with the module's bound."""
    q, K, V = (oracle.decode(x, "bf16") for x in (inp.q, inp.K, inp.V))
    kd, kt = oracle.k_from_rho(rho_d, D), oracle.k_from_rho(rho_t, L)
    idx_d = torch.full((B * Hq, kd), -1, dtype=torch.int32, device="cuda")
    idx_t = torch.full((B * Hq, kt), -1, dtype=torch.int32, device="cuda")
    lse = torch.empty(B * Hq, dtype=torch.float32, device="cuda")
    logits = torch.empty((B * Hq, L), dtype=torch.float32, device="cuda")
    O = R.rmm_decode_attention(bf16_tensor(inp.q), bf16_tensor(inp.K), bf16_tensor(inp.V), L, rho_d, rho_t,
                               out_dtype=torch.float32, idx_d=idx_d, idx_t=idx_t, lse=lse, logits=logits)
    assert R.rmm_device_error(clear=True) == 0
    got_d = idx_d.cpu().numpy().reshape(B, Hq, kd)
    got_t = idx_t.cpu().numpy().reshape(B, Hq, kt)
    got_s = logits.cpu().numpy().astype(np.float64).reshape(B, Hq, L)
    got_l = lse.cpu().numpy().astype(np.float64).reshape(B, Hq)
    got_o = to_f64(O)
    scale = 1.0 / math.sqrt(D)
    for b, h in heads:
        g = h * Hkv // Hq
        r = OD.decode_attention_head(q[b, h], K[b, g, :L], V[b, g, :L], rho_d, rho_t)
        np.testing.assert_array_equal(got_d[b, h], r["idx_d"])
        Id = r["idx_d"]
        absdot = scale * (np.abs(K[b, g, :L][:, Id]) @ np.abs(q[b, h, Id]))
        assert np.all(np.abs(got_s[b, h] - r["logits"]) <= D * 2.0 ** -24 * absdot * 1.01 + 1e-6)
        assert abs(got_l[b, h] - r["lse"]) <= 2e-5
        It = oracle.topk_indices(got_s[b, h], kt)
        np.testing.assert_array_equal(got_t[b, h], It)
        P = np.exp(r["logits"] - r["lse"])
        ref_o = oracle.reduced_matmul(P[None, :], V[b, g, :L], It)[0]
        bound = (kt * 2.0 ** -24 + 1e-5) * (P[It] @ np.abs(V[b, g, It])) + 1e-30
        assert np.all(np.abs(got_o[b, h] - ref_o) <= bound), (b, h)
    # without the optional outputs (the top-k writes only its bitmap): the same O
    O2 = R.rmm_decode_attention(bf16_tensor(inp.q), bf16_tensor(inp.K), bf16_tensor(inp.V), L, rho_d, rho_t,
                                out_dtype=torch.float32)
    assert torch.equal(O2, O)


def test_decode_attention_tied_logits():
    """Key rows repeating three patterns: each head's logits take three
    values, and the k_t boundary falls inside a run of equal logits, so only
    the lowest-index copies are kept (the top-k's compaction path, with and
    without the list output; clusters of 4 CTAs per head)."""
    B, Hq, Hkv, L, D = 1, 4, 1, 20000, 128
    inp = W.decode_attention(11, B, Hq, Hkv, L, D, 0.5, 0.5)
    inp.K[:, :, :L] = inp.K[:, :, np.arange(L) % 3]
    q, K, V = (oracle.decode(x, "bf16") for x in (inp.q, inp.K, inp.V))
    ref = OD.decode_attention(q, K, V, L, 0.5, 0.5)
    kt = oracle.k_from_rho(0.5, L)
    for h in range(Hq):   # the boundary splits a run of equal logits
        s = np.sort(ref["logits"][0, h])[::-1]
        assert s[kt - 1] == s[kt]
    idx_t = torch.full((Hq, kt), -1, dtype=torch.int32, device="cuda")
    O = R.rmm_decode_attention(bf16_tensor(inp.q), bf16_tensor(inp.K), bf16_tensor(inp.V), L, 0.5, 0.5,
                               out_dtype=torch.float32, idx_t=idx_t)
    np.testing.assert_array_equal(idx_t.cpu().numpy().reshape(B, Hq, kt), ref["idx_t"])
    assert rel_fro(to_f64(O), ref["O"]) <= 1e-5
    O2 = R.rmm_decode_attention(bf16_tensor(inp.q), bf16_tensor(inp.K), bf16_tensor(inp.V), L, 0.5, 0.5,
                                out_dtype=torch.float32)
    assert torch.equal(O2, O)
    assert R.rmm_device_error(clear=True) == 0


def test_decode_attention_full_size():
    """The benchmarked decode step (GQA 32/8 heads, D = 128, 32768 cached
    tokens, one sequence: token top-k on clusters of 4 CTAs), every head."""
    B, Hq, Hkv, L, D = 1, 32, 8, 32768, 128
    inp = W.decode_attention(5, B, Hq, Hkv, L, D, 0.5, 0.5)
    _check_own_selection(inp, B, Hq, Hkv, L, D, 0.5, 0.5, [(0, h) for h in range(Hq)])


def test_decode_attention_long_row():
    """A cache longer than eight top-k slices (8 x 51200 tokens): the token
    top-k takes the radix pass and the chunk starts come from the prefix
    kernel."""
    B, Hq, Hkv, L, D = 1, 2, 1, 8 * 51200 + 1, 64
    inp = W.decode_attention(7, B, Hq, Hkv, L, D, 0.5, 0.4)
    _check_own_selection(inp, B, Hq, Hkv, L, D, 0.5, 0.4, [(0, 0), (0, 1)])


def test_decode_attention_workspace_only_outputs():
    """No optional outputs: logits and token indices live in the workspace."""
    B, Hq, Hkv, L, D = 2, 4, 2, 640, 128
    inp = draw(B, Hq, Hkv, L, L, D, 0.5, 0.5)
    q, K, V = (oracle.decode(x, "bf16") for x in (inp.q, inp.K, inp.V))
    ref = OD.decode_attention(q, K, V, L, 0.5, 0.5)
    O = R.rmm_decode_attention(bf16_tensor(inp.q), bf16_tensor(inp.K), bf16_tensor(inp.V), L, 0.5, 0.5,
                               out_dtype=torch.float32)
    assert rel_fro(to_f64(O), ref["O"]) <= 1e-5
    assert R.rmm_device_error(clear=True) == 0


def test_decode_attention_rejects():
    q = torch.zeros((1, 4, 128), dtype=torch.bfloat16, device="cuda")
    K = torch.zeros((1, 2, 64, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(R.RMMError):          # L beyond the cache capacity
        R.rmm_decode_attention(q, K, K, 65, 0.5, 0.5)
    q96 = torch.zeros((1, 4, 96), dtype=torch.bfloat16, device="cuda")
    K96 = torch.zeros((1, 2, 64, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(R.RMMError):          # head_dim not 64 or 128
        R.rmm_decode_attention(q96, K96, K96, 64, 0.5, 0.5)
    q34 = torch.zeros((1, 34, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(R.RMMError):          # q-heads not a multiple of kv-heads
        R.rmm_decode_attention(q34, K, K, 64, 0.5, 0.5)
    q6 = torch.zeros((1, 6, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(R.RMMError):          # 3 q-heads per kv-head: not a supported group size
        R.rmm_decode_attention(q6, K, K, 64, 0.5, 0.5)
    assert R.rmm_device_error(clear=True) == 0
