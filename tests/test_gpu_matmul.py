"""GPU parity of the reduced-matmul path against the fp64 oracle, through the
C ABI: scores, top-k (bit-exact), compaction (exact), reduced GEMM (relative
Frobenius), the whole path on the seeded workloads, edge cases and the
device error word.

Tolerances: fp32 scores 1e-5 relative per element (squares are exact, the fp32
sum has a relative error of a few 1e-7); bf16 reduced GEMM with bf16 output:
every element within one bf16 ulp of the oracle and 2e-3 relative Frobenius
(outputs of >= 4096 elements); with fp32 output 1e-5 relative Frobenius (fp32
accumulation of exact bf16 products); fp32 SIMT GEMM 1e-5."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from oracle.conditioning import boundary_gaps, widen_topk_gaps
from tests.helpers import bf16_tensor, bf16_ulp, check_bf16_output, rel_fro, sample_rows, to_device, to_f64

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


def no_device_error():
    assert R.rmm_device_error(clear=True) == 0


# ------------------------------------------------------------------ score

@pytest.mark.parametrize("dtype,M,d", [("f32", 64, 256), ("bf16", 300, 777), ("bf16", 4096, 4096),
                                       ("bf16", 1, 9), ("bf16", 2049, 14336), ("f32", 513, 1003),
                                       ("bf16", 37, 8)])
def test_score_parity(dtype, M, d):
    if dtype == "f32":
        A = W.tiny_fp32(3, M=M, d=d, N=8).A
    else:
        A = W.llm_activation_bf16(7, M, d)
    At = to_device(A, dtype)
    ss = R.rmm_score(At)
    ref = oracle.column_sq_norms(oracle.decode(A, dtype))
    got = to_f64(ss)
    np.testing.assert_allclose(got, ref, rtol=1e-5, atol=0)
    s = R.rmm_score(At, sqrt_out=True)
    np.testing.assert_allclose(to_f64(s), np.sqrt(ref), rtol=1e-5)
    no_device_error()


def test_score_batched_and_strided():
    X = W.llm_activation_bf16(11, 5 * 700, 128).reshape(5, 700, 128)
    Xt = bf16_tensor(X)
    ss = R.rmm_score(Xt)
    for b in range(5):
        ref = oracle.column_sq_norms(oracle.decode(X[b], "bf16"))
        np.testing.assert_allclose(to_f64(ss[b]), ref, rtol=1e-5)
    # a column window of a wider matrix (lda > d, unaligned start -> scalar path)
    big = bf16_tensor(W.llm_activation_bf16(12, 200, 300))
    sub = big[:, 3:250]
    ss2 = R.rmm_score(sub)
    ref2 = oracle.column_sq_norms(to_f64(sub))
    np.testing.assert_allclose(to_f64(ss2), ref2, rtol=1e-5)
    # zero rows give zero scores
    z = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    assert torch.count_nonzero(R.rmm_score(z)).item() == 0
    no_device_error()


# ------------------------------------------------------------------ top-k

def _topk_cases():
    rng = np.random.default_rng(5)
    cases = []
    for d in (1, 7, 8, 33, 1000, 4096, 14336, 32768):
        s = rng.random(d).astype(np.float32) * 10
        for k in sorted({1, max(1, d // 2), max(1, (d * 7 + 9) // 10), d}):
            cases.append((f"rand d{d} k{k}", s, k))
    ties = np.zeros(100, np.float32)
    cases += [("all zero", ties, 37), ("all equal", np.full(257, 3.5, np.float32), 100)]
    s = rng.integers(0, 4, 5000).astype(np.float32)      # heavy ties at every boundary
    cases += [("ties k=1", s, 1), ("ties mid", s, 2500), ("ties k=d-1", s, 4999)]
    s = np.array([1.0, -0.0, 0.0, 2.0, 2.0, 1.0, 0.0, 2.0], np.float32)
    cases += [("signed zero", s, 6), ("dup boundary", s, 4)]
    s = np.arange(3000, dtype=np.float32)[::-1].copy()   # strictly decreasing
    cases += [("decreasing", s, 1234)]
    s = rng.random(12345).astype(np.float32)
    s[[10, 20, 30, 40]] = s.max() + 1                    # equal maxima, k inside them
    cases += [("top ties", s, 2)]
    s = (rng.random(2048).astype(np.float32) * 2 ** -126)  # subnormals
    cases += [("subnormal", s, 1024)]
    cases += [("negative", (rng.standard_normal(3001) * 5).astype(np.float32), 1500)]
    s = np.concatenate([np.float32([3e38, 1e-38]), rng.random(5000).astype(np.float32)])
    cases += [("wide range", s, 2000)]
    s = rng.random(51200).astype(np.float32)             # longest row one CTA could stage
    cases += [("staged max", s, 25600)]
    # rows split over a cluster of CTAs: equal keys on every slice boundary,
    # all keys equal (no histogram round), ragged last slices
    s = rng.integers(0, 3, 40001).astype(np.float32)
    cases += [("cluster ties", s, 13335), ("cluster ties k=1", s, 1)]
    cases += [("cluster all equal", np.full(40000, -2.5, np.float32), 12345)]
    s = rng.random(8 * 51200).astype(np.float32)         # longest row a cluster of eight stages
    cases += [("cluster max", s, 204800)]
    s = rng.random(8 * 51200 + 1).astype(np.float32)     # first row length re-read from global memory
    cases += [("global radix", s, 17)]
    return cases


@pytest.mark.parametrize("case", _topk_cases(), ids=lambda c: c[0])
def test_topk_bit_exact(case):
    _, s, k = case
    st = torch.from_numpy(s).cuda()
    got = R.rmm_topk(st, k).cpu().numpy()
    ref = oracle.topk_indices(s.astype(np.float64), k)
    np.testing.assert_array_equal(got, ref)
    no_device_error()


@pytest.mark.parametrize("rows,d,k", [(6, 20000, 2500),     # clusters of 4, rows not 16-byte aligned
                                      (40, 8192, 3000),     # clusters of 2
                                      (20, 30001, 9999),    # clusters of 4, ragged last slices
                                      (100, 3000, 1500)])   # one CTA per row
def test_topk_batched_rows(rows, d, k):
    rng = np.random.default_rng(9 + rows)
    S = rng.random((rows, d)).astype(np.float32)
    S[2] = np.round(S[2] * 3)
    pad = np.zeros((rows, d + 3), np.float32)
    pad[:, :d] = S
    st = torch.from_numpy(pad).cuda()[:, :d]
    out = torch.full((rows, k + 100), -7, dtype=torch.int32, device="cuda")
    R.rmm_topk(st, k, out=out[:, :k])
    got = out.cpu().numpy()
    for b in range(rows):
        np.testing.assert_array_equal(got[b, :k], oracle.topk_indices(S[b].astype(np.float64), k))
    assert np.all(got[:, k:] == -7)   # nothing written past k
    no_device_error()


# ------------------------------------------------------------------ compaction

@pytest.mark.parametrize("dtype,M,d,k", [("bf16", 300, 1000, 333), ("bf16", 4096, 4096, 2048),
                                         ("f32", 64, 256, 128), ("bf16", 3, 5, 1), ("bf16", 129, 2100, 2100)])
def test_compact_exact(dtype, M, d, k):
    rng = np.random.default_rng(M + d)
    A = W.llm_activation_bf16(3, M, d) if dtype == "bf16" else W.tiny_fp32(2, M=M, d=d, N=4).A
    idx = np.sort(rng.choice(d, k, replace=False)).astype(np.int32)
    At = to_device(A, dtype)
    it = torch.from_numpy(idx).cuda()
    AI = R.rmm_compact(At, it)
    np.testing.assert_array_equal(to_f64(AI), oracle.decode(A, dtype)[:, idx])
    no_device_error()


@pytest.mark.parametrize("M,d,lda,k", [(37, 60000, 60000, 30001),   # 120 KB rows: one staged row per block
                                       (19, 4096, 4104, 2048),      # padded pitch; last block of 3 rows
                                       (70, 1024, 1030, 700)])      # pitch not a multiple of 8: direct gather
def test_compact_staged_and_pitched(M, d, lda, k):
    rng = np.random.default_rng(M * 7 + d)
    A = W.llm_activation_bf16(11, M, d)
    buf = torch.zeros((M, lda), dtype=torch.bfloat16, device="cuda")
    buf[:, :d] = bf16_tensor(A)
    idx = np.sort(rng.choice(d, k, replace=False)).astype(np.int32)
    AI = R.rmm_compact(buf[:, :d], torch.from_numpy(idx).cuda())
    np.testing.assert_array_equal(to_f64(AI), oracle.decode(A, "bf16")[:, idx])
    no_device_error()


@pytest.mark.parametrize("M,d,N,k", [(300, 1000, 700, 333), (4096, 4096, 1024, 2048), (3, 5, 2, 1),
                                     (129, 2100, 701, 2100), (0, 64, 24, 10), (17, 96, 264, 65)])
def test_compact_gather_exact(M, d, N, k):
    """Both reduced operands in one launch equal A[:, I] and B[I, :] exactly."""
    rng = np.random.default_rng(M + d + N)
    A = W.llm_activation_bf16(5, max(M, 1), d)[:M]
    Bb = W.weight_bf16(6, d, N)
    idx = np.sort(rng.choice(d, k, replace=False)).astype(np.int32)
    At = bf16_tensor(A) if M > 0 else torch.empty((0, d), dtype=torch.bfloat16, device="cuda")
    Bt = _pitched(bf16_tensor(Bb))
    it = torch.from_numpy(idx).cuda()
    AI, BI = R.rmm_compact_gather(At, Bt, it)
    np.testing.assert_array_equal(to_f64(AI), oracle.decode(A, "bf16")[:, idx])
    np.testing.assert_array_equal(to_f64(BI), oracle.decode(Bb, "bf16")[idx, :])
    no_device_error()


def test_compact_gather_bad_index_gives_zeros_and_flag():
    M, d, N, k = 40, 128, 72, 16
    A = W.llm_activation_bf16(7, M, d)
    Bb = W.weight_bf16(8, d, N)
    idx = np.arange(k, dtype=np.int32)
    idx[3] = -2
    AI, BI = R.rmm_compact_gather(bf16_tensor(A), bf16_tensor(Bb), torch.from_numpy(idx).cuda())
    assert R.rmm_device_error(clear=True) == 1
    a, b = to_f64(AI), to_f64(BI)
    assert np.all(a[:, 3] == 0) and np.all(b[3] == 0)
    ok = np.delete(np.arange(k), 3)
    np.testing.assert_array_equal(a[:, ok], oracle.decode(A, "bf16")[:, idx[ok]])
    np.testing.assert_array_equal(b[ok], oracle.decode(Bb, "bf16")[idx[ok]])
    no_device_error()


# ------------------------------------------------------------------ reduced GEMM

def _pitched(t):
    """Same values in a buffer whose row pitch is a multiple of 8 elements
    (the bf16 kernel's documented layout rule); the logical width is unchanged."""
    n = t.shape[1]
    if n % 8 == 0:
        return t
    buf = torch.zeros((t.shape[0], (n + 7) // 8 * 8), dtype=t.dtype, device=t.device)
    buf[:, :n] = t
    return buf[:, :n]


GEMM_SHAPES = [
    (128, 256, 256, 64),      # one tile, one k block
    (300, 1000, 700, 333),    # ragged M, N, k
    (1, 64, 8, 1),            # degenerate
    (17, 96, 264, 65),        # N just past a tile, k just past a block
    (512, 4096, 1024, 2048),  # several tiles and k blocks
    (1000, 3000, 2000, 1500),
    (1024, 1024, 7424, 512),  # 116 tiles of 256 x 256: a last wave too full to split into halves
]


@pytest.mark.parametrize("M,d,N,k", GEMM_SHAPES)
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_gemm_bf16_parity(M, d, N, k, out_dtype):
    inp = W.scaled_matmul_bf16(21, M, d, N)
    rng = np.random.default_rng(k)
    idx = np.sort(rng.choice(d, k, replace=False)).astype(np.int32)
    A = oracle.decode(inp.A, "bf16")
    Bm = oracle.decode(inp.B, "bf16")
    ref = oracle.reduced_matmul(A, Bm, idx)
    At = bf16_tensor(inp.A)
    Bt = _pitched(bf16_tensor(inp.B))
    it = torch.from_numpy(idx).cuda()
    AI = R.rmm_compact(At, it)
    Y = R.rmm_gemm(AI, Bt, it, out_dtype=out_dtype)
    if out_dtype == torch.bfloat16:
        absprod = oracle.reduced_matmul(np.abs(A), np.abs(Bm), idx)
        check_bf16_output(to_f64(Y), ref, absprod, k)
    else:
        assert rel_fro(to_f64(Y), ref) <= 1e-5
    no_device_error()


def _fused_first_cols(M, N):
    """Columns of B_I copied before the CTA-pair product starts, as the library
    plans it (the column blocks its first wave of tiles reads); the product's
    own warps copy the rest.  Mirrors the host rule so that each case below is
    known to exercise the copy inside the product."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    pairs = sms // 2
    num_m, num_n = (M + 255) // 256, (N + 255) // 256
    tiles = num_m * num_n
    rem = tiles % pairs
    split_from = tiles - rem if (rem > 0 and 2 * rem <= pairs) else tiles
    items = split_from + 2 * (tiles - split_from)
    first = min(items, pairs) - 1
    tile = first if first < split_from else split_from + (first - split_from) // 2
    return min((tile // num_m + 1) * 256, N)


FUSED_SHAPES = [  # M, d, N, k: M >= 256, N a multiple of 8, more tiles than one wave
    (20480, 256, 512, 33),     # one column block copied inside; 3 row units, the last of one row
    (16384, 600, 776, 257),    # two blocks inside, the last 8 columns wide; ragged units
    (2048, 4096, 4104, 4096),  # every row kept; 7 of 17 blocks inside
]


@pytest.mark.parametrize("M,d,N,k", FUSED_SHAPES)
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_gemm_fused_gather_parity(M, d, N, k, out_dtype):
    """The product kernel that fills part of B_I with its own warps: the same
    bounds as the two-launch form, on a workspace filled with 0xFF bytes (the
    call must zero its counters), called twice on that workspace with
    different index sets."""
    assert _fused_first_cols(M, N) < N
    inp = W.scaled_matmul_bf16(23 + M % 1000, M, d, N)
    A = oracle.decode(inp.A, "bf16")
    Bm = oracle.decode(inp.B, "bf16")
    At = bf16_tensor(inp.A)
    Bt = bf16_tensor(inp.B)
    ws = torch.full((R.rmm_gemm_workspace_size(R.RMM_BF16, N, k),), 0xFF, dtype=torch.uint8, device="cuda")
    for trial in range(2):
        rng = np.random.default_rng(k + 17 * trial)
        idx = np.sort(rng.choice(d, k, replace=False)).astype(np.int32)
        it = torch.from_numpy(idx).cuda()
        Y = R.rmm_gemm(R.rmm_compact(At, it), Bt, it, out_dtype=out_dtype, ws=ws)
        ref = oracle.reduced_matmul(A, Bm, idx)
        if out_dtype == torch.bfloat16:
            check_bf16_output(to_f64(Y), ref, oracle.reduced_matmul(np.abs(A), np.abs(Bm), idx), k)
        else:
            assert rel_fro(to_f64(Y), ref) <= 1e-5
        no_device_error()


def test_gemm_fused_gather_bad_index_flagged():
    """An out-of-range kept row: zero in both parts of B_I (the column block
    copied ahead and the one the product copies), the error word set, the
    rest of the product exact to the usual bound."""
    M, d, N, k, bad = 20480, 256, 512, 64, 40
    assert _fused_first_cols(M, N) < N
    inp = W.scaled_matmul_bf16(29, M, d, N)
    idx = np.arange(k, dtype=np.int32) * 3
    idx[bad] = d + 5
    it = torch.from_numpy(idx).cuda()
    AI = R.rmm_compact(bf16_tensor(inp.A), it)
    assert R.rmm_device_error(clear=True) == 1
    Y = R.rmm_gemm(AI, bf16_tensor(inp.B), it, out_dtype=torch.float32)
    assert R.rmm_device_error(clear=True) == 1
    good = np.delete(np.arange(k), bad)
    ref = to_f64(AI)[:, good] @ oracle.decode(inp.B, "bf16")[idx[good]]
    assert rel_fro(to_f64(Y), ref) <= 1e-5
    no_device_error()


DECODE_SHAPES = [  # M, d, N, k: a few activation rows (decode); kept rows of B read in place
    (1, 4096, 4096, 2048),
    (2, 1000, 700, 333),       # ragged N and k
    (3, 512, 8, 1),            # one kept row
    (5, 4096, 1032, 4096),     # every row kept
    (8, 2048, 14336, 1024),
    (13, 4096, 264, 2867),
    (16, 4096, 4096, 2048),
]


@pytest.mark.parametrize("M,d,N,k", DECODE_SHAPES)
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_gemm_few_rows_parity(M, d, N, k, out_dtype):
    inp = W.scaled_matmul_bf16(31 + M, M, d, N)
    rng = np.random.default_rng(M * 11 + k)
    idx = np.sort(rng.choice(d, k, replace=False)).astype(np.int32)
    A = oracle.decode(inp.A, "bf16")
    Bm = oracle.decode(inp.B, "bf16")
    At, Bt = bf16_tensor(inp.A), _pitched(bf16_tensor(inp.B))
    it = torch.from_numpy(idx).cuda()
    AI = R.rmm_compact(At, it)
    Y = R.rmm_gemm(AI, Bt, it, out_dtype=out_dtype)
    ref = A[:, idx] @ Bm[idx, :]
    if out_dtype == torch.float32:
        # fp32 sums of exact bf16 products, k terms in some order
        bound = k * 2.0 ** -24 * (np.abs(A[:, idx]) @ np.abs(Bm[idx, :])) + 1e-30
        assert np.all(np.abs(to_f64(Y) - ref) <= bound)
    else:
        check_bf16_output(to_f64(Y), ref, np.abs(A[:, idx]) @ np.abs(Bm[idx, :]), k)
    no_device_error()


def test_gemm_few_rows_bad_index_flagged():
    M, d, N, k = 4, 256, 128, 64
    inp = W.scaled_matmul_bf16(77, M, d, N)
    idx = np.arange(k, dtype=np.int32)
    idx[9] = d + 5
    At, Bt = bf16_tensor(inp.A), bf16_tensor(inp.B)
    it = torch.from_numpy(idx).cuda()
    AI = R.rmm_compact(At, it)
    assert R.rmm_device_error(clear=True) == 1
    R.rmm_gemm(AI, Bt, it, out_dtype=torch.float32)
    assert R.rmm_device_error(clear=True) == 1
    no_device_error()


@pytest.mark.parametrize("M", [1, 4, 16])
def test_path_decode_rows(M):
    """Whole path at decode sizes on the MLP up/gate and down shapes."""
    for inp in (W.llm_activation_bf16(41 + M, M, 4096), W.llm_activation_bf16(43 + M, M, 14336)):
        d = inp.shape[1]
        Wb = W.weight_bf16(5, d, 4096 if d == 14336 else 14336)
        A = oracle.decode(inp, "bf16")
        Bm = oracle.decode(Wb, "bf16")
        cond, _ = widen_topk_gaps(inp, "bf16", [oracle.k_from_rho(0.5, d)])
        Ac = oracle.decode(cond, "bf16")
        k = oracle.k_from_rho(0.5, d)
        idx = oracle.topk_indices(oracle.column_sq_norms(Ac), k)
        idx_out = torch.empty(k, dtype=torch.int32, device="cuda")
        ss_out = torch.empty(d, dtype=torch.float32, device="cuda")
        Y = R.rmm_matmul(bf16_tensor(cond), bf16_tensor(Wb), 0.5, idx_out=idx_out, ss_out=ss_out)
        np.testing.assert_array_equal(idx_out.cpu().numpy(), idx)
        np.testing.assert_allclose(to_f64(ss_out), oracle.column_sq_norms(Ac), rtol=1e-5)
        ref = Ac[:, idx] @ Bm[idx, :]
        check_bf16_output(to_f64(Y), ref, np.abs(Ac[:, idx]) @ np.abs(Bm[idx, :]), k)
    no_device_error()


@pytest.mark.parametrize("M,d,N,rho,ties", [(2, 1000, 777, 0.37, False), (3, 22528, 512, 0.9, False),
                                             (1, 64, 8, 1.0, False), (4, 4096, 1000, 0.5, True),
                                             (1, 2048, 4104, 0.25, True), (8, 4096, 2048, 0.5, False),
                                             (13, 1024, 296, 0.6, True), (16, 19072, 512, 0.5, False)])
def test_path_decode_fused_selection(M, d, N, rho, ties):
    """Up to 16 rows with d a multiple of 8 run the product whose CTAs each make
    the selection themselves: the index list, the scores and Y against the
    oracle, including heavy ties (groups of equal columns: lowest index wins),
    rho = 1 and ragged N."""
    bits = W.llm_activation_bf16(300 + M + d, M, d)
    if ties:
        bits = bits.copy()
        bits[:, 1::4] = bits[:, 0::4][:, : bits[:, 1::4].shape[1]]  # every 4th pair of columns equal
        bits[:, 2::4] = bits[:, 0::4][:, : bits[:, 2::4].shape[1]]
    k = oracle.k_from_rho(rho, d)
    if not ties:
        bits, _ = widen_topk_gaps(bits, "bf16", [k])
    A = oracle.decode(bits, "bf16")
    Wb = W.weight_bf16(6, d, N)
    Bm = oracle.decode(Wb, "bf16")
    idx_out = torch.full((k,), -1, dtype=torch.int32, device="cuda")
    ss_out = torch.empty(d, dtype=torch.float32, device="cuda")
    Y = R.rmm_matmul(bf16_tensor(bits), _pitched(bf16_tensor(Wb)), rho, idx_out=idx_out, ss_out=ss_out,
                     out_dtype=torch.float32)
    np.testing.assert_allclose(to_f64(ss_out), oracle.column_sq_norms(A), rtol=1e-5)
    # with ties the set is defined on the scores as computed (equal columns
    # give equal fp32 sums): the oracle's top-k of the GPU's own scores; else
    # the oracle's scores, whose boundary gap was widened
    idx = oracle.topk_indices(to_f64(ss_out) if ties else oracle.column_sq_norms(A), k)
    np.testing.assert_array_equal(idx_out.cpu().numpy(), idx)
    ref = A[:, idx] @ Bm[idx, :]
    bound = k * 2.0 ** -24 * (np.abs(A[:, idx]) @ np.abs(Bm[idx, :])) + 1e-30
    assert np.all(np.abs(to_f64(Y) - ref) <= bound)
    no_device_error()


def test_path_decode_unaligned_rows():
    """Few rows with a row pitch that is not a multiple of 8 (the fused
    selection's scalar path) and d not a multiple of 8."""
    M, d, N, rho = 3, 1001, 264, 0.4
    A_bits = W.llm_activation_bf16(91, M, d)
    k = oracle.k_from_rho(rho, d)
    cond, _ = widen_topk_gaps(A_bits, "bf16", [k])
    Ac = oracle.decode(cond, "bf16")
    Wb = W.weight_bf16(92, d, N)
    Bm = oracle.decode(Wb, "bf16")
    buf = torch.zeros((M, d + 2), dtype=torch.bfloat16, device="cuda")
    buf[:, :d] = bf16_tensor(cond)
    idx_out = torch.empty(k, dtype=torch.int32, device="cuda")
    Y = R.rmm_matmul(buf[:, :d], _pitched(bf16_tensor(Wb)), rho, idx_out=idx_out)
    idx = oracle.topk_indices(oracle.column_sq_norms(Ac), k)
    np.testing.assert_array_equal(idx_out.cpu().numpy(), idx)
    check_bf16_output(to_f64(Y), Ac[:, idx] @ Bm[idx, :], np.abs(Ac[:, idx]) @ np.abs(Bm[idx, :]), k)
    no_device_error()


def test_gemm_writes_only_its_window():
    """Guard bands: Y is a window of a larger buffer; nothing outside changes."""
    M, d, N, k = 200, 640, 300, 200
    inp = W.scaled_matmul_bf16(22, M, d, N)
    idx = np.sort(np.random.default_rng(1).choice(d, k, replace=False)).astype(np.int32)
    At, Bt = bf16_tensor(inp.A), _pitched(bf16_tensor(inp.B))
    it = torch.from_numpy(idx).cuda()
    AI = R.rmm_compact(At, it)
    big = torch.full((M + 2, 320), 7.0, dtype=torch.float32, device="cuda")
    Y = big[1:M + 1, 8:8 + N]
    R.rmm_gemm(AI, Bt, it, out=Y)
    ref = oracle.reduced_matmul(oracle.decode(inp.A, "bf16"), oracle.decode(inp.B, "bf16"), idx)
    assert rel_fro(to_f64(Y), ref) <= 1e-5
    b = big.cpu().numpy()
    mask = np.ones_like(b, dtype=bool)
    mask[1:M + 1, 8:8 + N] = False
    assert np.all(b[mask] == 7.0)
    no_device_error()


def test_gemm_f32_tiny_workload():
    inp = W.tiny_fp32(0)
    Y, idx, _ = oracle.rmm_path(oracle.decode(inp.A, "f32"), oracle.decode(inp.B, "f32"), 0.5)
    At, Bt = to_device(inp.A, "f32"), to_device(inp.B, "f32")
    it = torch.from_numpy(idx.astype(np.int32)).cuda()
    got = R.rmm_gemm(R.rmm_compact(At, it), Bt, it)
    assert rel_fro(to_f64(got), Y) <= 1e-5
    no_device_error()


def test_bad_index_is_flagged_not_read():
    M, d, N, k = 64, 128, 64, 16
    inp = W.scaled_matmul_bf16(23, M, d, N)
    idx = np.arange(k, dtype=np.int32)
    idx[5] = d + 1000
    At, Bt = bf16_tensor(inp.A), bf16_tensor(inp.B)
    it = torch.from_numpy(idx).cuda()
    AI = R.rmm_compact(At, it)
    assert R.rmm_device_error(clear=True) == 1
    R.rmm_gemm(AI, Bt, it)
    assert R.rmm_device_error(clear=True) == 1
    no_device_error()


# ------------------------------------------------------------------ whole path on the workloads

def _check_path(inp, rho, rows=None, out_dtype=torch.bfloat16, cond=None):
    A_bits = cond if cond is not None else inp.A
    A = oracle.decode(A_bits, inp.dtype)
    Bm = oracle.decode(inp.B, inp.dtype)
    ss = oracle.column_sq_norms(A)
    k = oracle.k_from_rho(rho, A.shape[1])
    idx = oracle.topk_indices(ss, k)
    At = to_device(A_bits, inp.dtype)
    Bt = to_device(inp.B, inp.dtype)
    idx_out = torch.empty(k, dtype=torch.int32, device="cuda")
    ss_out = torch.empty(A.shape[1], dtype=torch.float32, device="cuda")
    if inp.dtype == "f32":
        out_dtype = torch.float32
    Y = R.rmm_matmul(At, Bt, rho, out_dtype=out_dtype, idx_out=idx_out, ss_out=ss_out)
    np.testing.assert_array_equal(idx_out.cpu().numpy(), idx)
    np.testing.assert_allclose(to_f64(ss_out), ss, rtol=1e-5)
    rows = np.arange(A.shape[0]) if rows is None else rows
    ref = A[rows][:, idx] @ Bm[idx, :]
    if out_dtype == torch.float32:
        err = rel_fro(to_f64(Y)[rows], ref)
        assert err <= 1e-5, err
    else:
        absprod = np.abs(A[rows][:, idx]) @ np.abs(Bm[idx, :])
        err = check_bf16_output(to_f64(Y)[rows], ref, absprod, k)
    no_device_error()
    return err


def test_path_tiny_fp32_workload():
    inp = W.tiny_fp32(0)
    A2, _ = widen_topk_gaps(inp.A, "f32", [128])
    _check_path(inp, 0.5, cond=A2)


@pytest.mark.parametrize("rho", [0.5, 0.7, 0.8, 1.0])
def test_path_mlp_up_small(rho):
    inp = W.mlp_up(seed=1, tokens=512, hidden=1024, ffn=1536)
    ks = [oracle.k_from_rho(r, 1024) for r in inp.rhos]
    A2, _ = widen_topk_gaps(inp.A, "bf16", ks)
    _check_path(inp, rho, cond=A2)


@pytest.mark.parametrize("rho", [0.5, 0.7, 0.8, 1.0])
def test_path_mlp_up_full(rho):
    """MLP up/gate projection 4096 x 4096 x 14336 bf16, all quoted rho."""
    inp = _full("up")
    _check_path(inp, rho, rows=sample_rows(inp.M), cond=_full_cond("up"))


@pytest.mark.parametrize("rho", [0.5, 0.8, 1.0])
def test_path_mlp_down_full(rho):
    """MLP down projection 4096 x 14336 x 4096 bf16, all quoted rho."""
    inp = _full("down")
    _check_path(inp, rho, rows=sample_rows(inp.M), cond=_full_cond("down"))


_CACHE = {}


def _full(which):
    if which not in _CACHE:
        _CACHE.clear()
        _CACHE[which] = W.mlp_up() if which == "up" else W.mlp_down()
    return _CACHE[which]


def _full_cond(which):
    key = which + "_cond"
    if key not in _CACHE:
        inp = _full(which)
        ks = [oracle.k_from_rho(r, inp.d) for r in inp.rhos]
        _CACHE[key], _ = widen_topk_gaps(inp.A, "bf16", ks)
    return _CACHE[key]


# ------------------------------------------------------------------ 70B-shaped layer

@pytest.mark.slow
@pytest.mark.parametrize("which", ["q_proj", "k_proj", "up_proj", "down_proj"])
def test_path_layer70b(which):
    """The 70B-shaped layer's distinct projection shapes (q/o 2048x8192x8192,
    k/v 2048x8192x1024 at rho 0.5; up/gate 2048x8192x28672 and down
    2048x28672x8192 at rho 0.8), whole path, sampled rows."""
    inp = W.layer70b_inputs(which)
    ks = [oracle.k_from_rho(r, inp.d) for r in inp.rhos]
    A2, _ = widen_topk_gaps(inp.A, "bf16", ks)
    _check_path(inp, inp.rhos[0], rows=sample_rows(inp.M), cond=A2)


# ------------------------------------------------------------------ int8 weight (weight-only quantisation)

def _pitched16(t):
    """int8 matrix in a buffer whose row pitch is a multiple of 16 bytes."""
    n = t.shape[1]
    if n % 16 == 0:
        return t
    buf = torch.zeros((t.shape[0], (n + 15) // 16 * 16), dtype=t.dtype, device=t.device)
    buf[:, :n] = t
    return buf[:, :n]


def _check_w8(got, A_I, q_I, s, k, out_dtype):
    """Oracle comparison for A_I · (q_I * s): the products a*q are exact in fp32
    (8 + 7 significant bits), the k-term fp32 sum and the scale multiply add
    at most (k + 1) * 2^-24 * sum |a q s| per element."""
    ref = A_I @ (q_I.astype(np.float64) * s.astype(np.float64)[None, :])
    absprod = np.abs(A_I) @ (np.abs(q_I.astype(np.float64)) * s.astype(np.float64)[None, :])
    if out_dtype == torch.float32:
        bound = (k + 1) * 2.0 ** -24 * absprod + 1e-30
        assert np.all(np.abs(got - ref) <= bound)
        if got.size >= 4096:
            assert rel_fro(got, ref) <= 1e-5
        return
    check_bf16_output(got, ref, absprod, k + 1)


W8_SHAPES = [  # M, d, N, k
    (1, 4096, 4096, 2048),     # decode: kept int8 rows read in place
    (3, 1000, 700, 333),       # ragged N (pitched rows) and k
    (8, 2048, 14336, 1024),
    (16, 4096, 4096, 2048),
    (17, 96, 272, 65),         # tensor-core path: N just past a tile, k just past a block
    (300, 1000, 700, 333),     # ragged M, N, k
    (512, 4096, 1024, 2048),   # CTA-pair tensor-core path
]


@pytest.mark.parametrize("M,d,N,k", W8_SHAPES)
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_gemm_w8_parity(M, d, N, k, out_dtype):
    A_bits = W.llm_activation_bf16(61 + M, M, d)
    q, s = W.weight_int8(62 + M, d, N)
    rng = np.random.default_rng(M * 7 + k)
    idx = np.sort(rng.choice(d, k, replace=False)).astype(np.int32)
    A = oracle.decode(A_bits, "bf16")
    it = torch.from_numpy(idx).cuda()
    AI = R.rmm_compact(bf16_tensor(A_bits), it)
    qt = _pitched16(torch.from_numpy(q).cuda())
    st = torch.from_numpy(s).cuda()
    Y = R.rmm_gemm_w8(AI, qt, st, it, out_dtype=out_dtype)
    _check_w8(to_f64(Y), A[:, idx], q[idx], s, k, out_dtype)
    # the oracle's own int8 product agrees with the check's reference
    np.testing.assert_allclose(oracle.reduced_matmul_w8(A, q, s, idx),
                               A[:, idx] @ (q[idx].astype(np.float64) * s.astype(np.float64)), rtol=1e-12)
    no_device_error()


@pytest.mark.parametrize("M", [1, 16, 300])
def test_path_w8(M):
    """Whole path with an int8 weight: selection bit-exact, product within bounds."""
    d, N, rho = 4096, 1040, 0.5
    A_bits = W.llm_activation_bf16(71 + M, M, d)
    k = oracle.k_from_rho(rho, d)
    cond, _ = widen_topk_gaps(A_bits, "bf16", [k])
    Ac = oracle.decode(cond, "bf16")
    q, s = W.weight_int8(72, d, N)
    idx_out = torch.empty(k, dtype=torch.int32, device="cuda")
    Y = R.rmm_matmul_w8(bf16_tensor(cond), torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda(), rho,
                        idx_out=idx_out)
    Yo, idx, _ = oracle.rmm_w8(Ac, q, s, rho)
    np.testing.assert_array_equal(idx_out.cpu().numpy(), idx)
    _check_w8(to_f64(Y), Ac[:, idx], q[idx], s, k, torch.bfloat16)
    assert rel_fro(to_f64(Y), Yo) <= 2e-3
    no_device_error()


def test_path_w8_mlp_up_full():
    """MLP up/gate projection 4096 x 4096 x 14336 with an int8 weight at rho = 0.5,
    the launch configuration the benchmark times; sampled rows vs the oracle."""
    inp = W.mlp_up_w8()
    k = oracle.k_from_rho(0.5, inp.d)
    cond, _ = widen_topk_gaps(inp.A, "bf16", [k])
    Ac = oracle.decode(cond, "bf16")
    q, s = inp.B, inp.meta["b_scale"]
    idx_out = torch.empty(k, dtype=torch.int32, device="cuda")
    Y = R.rmm_matmul_w8(bf16_tensor(cond), torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda(), 0.5,
                        idx_out=idx_out)
    idx = oracle.topk_indices(oracle.column_sq_norms(Ac), k)
    np.testing.assert_array_equal(idx_out.cpu().numpy(), idx)
    rows = sample_rows(inp.M)
    _check_w8(to_f64(Y)[rows], Ac[rows][:, idx], q[idx], s, k, torch.bfloat16)
    no_device_error()


@pytest.mark.parametrize("M", [2, 200, 20480])  # in-place rows, gather launch, copy inside the product
def test_gemm_w8_bad_index_flagged(M):
    d, N, k = 256, 512, 64
    if M >= 256:
        assert _fused_first_cols(M, N) < N
    A_bits = W.llm_activation_bf16(81, M, d)
    q, s = W.weight_int8(82, d, N)
    idx = np.arange(k, dtype=np.int32)
    idx[5] = d + 3
    it = torch.from_numpy(idx).cuda()
    AI = R.rmm_compact(bf16_tensor(A_bits), it)
    assert R.rmm_device_error(clear=True) == 1
    Y = R.rmm_gemm_w8(AI, torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda(), it, out_dtype=torch.float32)
    assert R.rmm_device_error(clear=True) == 1
    # the bad index contributes nothing; the rest is the product over the good ones
    good = np.delete(np.arange(k), 5)
    A = oracle.decode(A_bits, "bf16")
    _check_w8(to_f64(Y), to_f64(AI)[:, good], q[idx[good]], s, k, torch.float32)
    no_device_error()


def test_gemm_w8_rejects_bad_layouts():
    A_I = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    it = torch.arange(64, dtype=torch.int32, device="cuda")
    s = torch.ones(24, dtype=torch.float32, device="cuda")
    q = torch.zeros((128, 24), dtype=torch.int8, device="cuda")   # row pitch 24 bytes
    with pytest.raises(R.RMMError):
        R.rmm_gemm_w8(A_I, q, s, it)
    with pytest.raises(ValueError):
        R.rmm_gemm_w8(A_I, _pitched16(q), s[:10], it)
    with pytest.raises(TypeError):
        R.rmm_gemm_w8(A_I, _pitched16(q).to(torch.int16), s, it)
    no_device_error()


# ------------------------------------------------------------------ block driver

@pytest.mark.parametrize("M", [5, 300, 1024, 20480])
def test_matmul_multi_shared_selection(M):
    """q/k/v-style products on one activation: one index set, every product
    against the oracle.  At 20480 rows the first and third products copy
    part of their B_I inside the product kernel and the second does not."""
    d, Ns, rho = 1024, (512, 128, 264), 0.5
    if M == 20480:
        assert [_fused_first_cols(M, n) < n for n in Ns] == [True, False, True]
    A_bits = W.llm_activation_bf16(101 + M, M, d)
    k = oracle.k_from_rho(rho, d)
    cond, _ = widen_topk_gaps(A_bits, "bf16", [k])
    Ac = oracle.decode(cond, "bf16")
    Wb = [W.weight_bf16(102, d, n, group=i) for i, n in enumerate(Ns)]
    Bm = [oracle.decode(w, "bf16") for w in Wb]
    idx_out = torch.empty(k, dtype=torch.int32, device="cuda")
    Ys = R.rmm_matmul_multi(bf16_tensor(cond), [_pitched(bf16_tensor(w)) for w in Wb], rho, idx_out=idx_out)
    refs, idx, _ = oracle.block.matmul_shared(Ac, Bm, rho)
    np.testing.assert_array_equal(idx_out.cpu().numpy(), idx)
    for Y, ref, B in zip(Ys, refs, Bm):
        check_bf16_output(to_f64(Y), ref, np.abs(Ac[:, idx]) @ np.abs(B[idx, :]), k)
    no_device_error()


def test_matmul_multi_given_scores():
    """Selection from caller-given scores (no score pass)."""
    M, d, N, rho = 64, 512, 256, 0.3
    A_bits = W.llm_activation_bf16(111, M, d)
    k = oracle.k_from_rho(rho, d)
    cond, _ = widen_topk_gaps(A_bits, "bf16", [k])
    Ac = oracle.decode(cond, "bf16")
    ss = oracle.column_sq_norms(Ac)
    Wb = W.weight_bf16(112, d, N)
    idx_out = torch.empty(k, dtype=torch.int32, device="cuda")
    (Y,) = R.rmm_matmul_multi(bf16_tensor(cond), [bf16_tensor(Wb)], rho, idx_out=idx_out,
                              ss_in=torch.from_numpy(ss.astype(np.float32)).cuda())
    idx = oracle.topk_indices(ss, k)
    np.testing.assert_array_equal(idx_out.cpu().numpy(), idx)
    Bm = oracle.decode(Wb, "bf16")
    check_bf16_output(to_f64(Y), Ac[:, idx] @ Bm[idx, :], np.abs(Ac[:, idx]) @ np.abs(Bm[idx, :]), k)
    no_device_error()


def _gate_up(seed, M, N):
    rng = np.random.default_rng(seed)
    G = W.f32_to_bf16_bits(rng.standard_normal((M, N)) * 2.0)
    U = W.f32_to_bf16_bits(rng.standard_normal((M, N)))
    return G, U


@pytest.mark.parametrize("M,N", [(300, 1000), (4096, 2048), (7, 13)])
def test_silu_mul_score(M, N):
    """H within one bf16 ulp of the oracle (fp32 SiLU rounds differently near
    a bf16 rounding boundary, so a few elements may differ by one ulp); the
    fused scores are the column scores of the H the kernel stored (exact
    squares, fp32 sums: rtol 1e-5)."""
    G, U = _gate_up(120 + M, M, N)
    Gt, Ut = bf16_tensor(G), bf16_tensor(U)
    if N % 8:
        Gt, Ut = _pitched(Gt), _pitched(Ut)
    H = torch.zeros((M, (N + 7) // 8 * 8), dtype=torch.bfloat16, device="cuda")[:, :N]
    H, ss = R.rmm_silu_mul_score(Gt, Ut, out=H)
    ref = oracle.block.silu_mul_bf16(oracle.decode(G, "bf16"), oracle.decode(U, "bf16"))
    got = to_f64(H)
    diff = np.abs(got - ref)
    assert np.all(diff <= bf16_ulp(ref) + 1e-30)
    assert np.mean(diff > 0) < 1e-3
    np.testing.assert_allclose(to_f64(ss), oracle.column_sq_norms(got), rtol=1e-5, atol=1e-30)
    no_device_error()


@pytest.mark.parametrize("M", [4, 512])
def test_mlp_block(M):
    """The gated MLP block end to end, checked stage by stage on the GPU's own
    intermediates.  rmm_mlp_block is rmm_matmul_multi (up, gate), then
    rmm_silu_mul_score, then rmm_matmul_multi (down) from the fused scores, so
    the same public calls give it bit for bit; from them:
      - the up/gate selection reads X (gaps widened): bit-exact;
      - U and G: every element within one bf16 ulp plus the fp32-sum bound of
        the oracle's reduced product on that selection;
      - H: within one bf16 ulp of the oracle's SiLU(G) * U on the GPU's G, U;
        its scores are the column scores of that H (rtol 1e-5);
      - the down selection is the top-k of those scores (bit-exact where the
        boundary gap is clear, else every swapped index within 1e-5);
      - Y: every element within the bf16 bound of the oracle's reduced product
        H[:, J] W_down[J, :] on the GPU's H and J, relative Frobenius <= 2e-3.
    Against the oracle's whole block (fp64 all the way): identical up/gate
    set, down-set swaps only within 1e-3 of its boundary score, and Y within
    2e-3 relative Frobenius when the down sets agree."""
    dm, dff, rho_up, rho_down = 1024, 2816, 0.8, 0.5
    X_bits = W.llm_activation_bf16(130 + M, M, dm)
    ku = oracle.k_from_rho(rho_up, dm)
    cond, _ = widen_topk_gaps(X_bits, "bf16", [ku])
    Xc = oracle.decode(cond, "bf16")
    Wu = W.weight_bf16(131, dm, dff, group=0)
    Wg = W.weight_bf16(131, dm, dff, group=1)
    Wd = W.weight_bf16(131, dff, dm, group=2)
    Wu_f, Wg_f, Wd_f = (oracle.decode(w, "bf16") for w in (Wu, Wg, Wd))
    kd = oracle.k_from_rho(rho_down, dff)
    Xt, Wut, Wgt, Wdt = (bf16_tensor(x) for x in (cond, Wu, Wg, Wd))
    idx_up = torch.empty(ku, dtype=torch.int32, device="cuda")
    idx_down = torch.empty(kd, dtype=torch.int32, device="cuda")
    Y = R.rmm_mlp_block(Xt, Wut, Wgt, Wdt, rho_up, rho_down, idx_up=idx_up, idx_down=idx_down)
    # the same chain through the public calls, keeping the intermediates
    ldf = (dff + 7) // 8 * 8
    Ut = torch.empty((M, ldf), dtype=torch.bfloat16, device="cuda")[:, :dff]
    Gt = torch.empty((M, ldf), dtype=torch.bfloat16, device="cuda")[:, :dff]
    Ht = torch.empty((M, ldf), dtype=torch.bfloat16, device="cuda")[:, :dff]
    I_t = torch.empty(ku, dtype=torch.int32, device="cuda")
    J_t = torch.empty(kd, dtype=torch.int32, device="cuda")
    R.rmm_matmul_multi(Xt, [Wut, Wgt], rho_up, outs=[Ut, Gt], idx_out=I_t)
    Ht, ssH = R.rmm_silu_mul_score(Gt, Ut, out=Ht)
    (Y2,) = R.rmm_matmul_multi(Ht, [Wdt], rho_down, ss_in=ssH, idx_out=J_t)
    assert torch.equal(Y, Y2) and torch.equal(idx_up, I_t) and torch.equal(idx_down, J_t)
    I = idx_up.cpu().numpy()
    J = idx_down.cpu().numpy()
    # up / gate
    I_ref = oracle.topk_indices(oracle.column_sq_norms(Xc), ku)
    np.testing.assert_array_equal(I, I_ref)
    for got_t, Wf in ((Ut, Wu_f), (Gt, Wg_f)):
        check_bf16_output(to_f64(got_t), oracle.reduced_matmul(Xc, Wf, I),
                          oracle.reduced_matmul(np.abs(Xc), np.abs(Wf), I), ku)
    # H and its scores
    U_g, G_g, H_g = to_f64(Ut), to_f64(Gt), to_f64(Ht)
    H_ref = oracle.block.silu_mul_bf16(G_g, U_g)
    assert np.all(np.abs(H_g - H_ref) <= bf16_ulp(H_ref) + 1e-30)
    ss_h = oracle.column_sq_norms(H_g)
    np.testing.assert_allclose(to_f64(ssH), ss_h, rtol=1e-5, atol=1e-30)
    # down selection: the top-k of the scores of the stored H
    gap, _ = boundary_gaps(ss_h, [kd])
    J_ref = oracle.topk_indices(ss_h, kd)
    if gap[kd] >= 2e-5:
        np.testing.assert_array_equal(J, J_ref)
    else:
        thr = np.sort(ss_h)[::-1][kd - 1]
        sw = np.setxor1d(J, J_ref)
        assert np.all(np.abs(ss_h[sw] - thr) <= 1e-5 * thr), (sw, thr)
    # Y against the oracle's product on the GPU's own H and J
    check_bf16_output(to_f64(Y), oracle.reduced_matmul(H_g, Wd_f, J), oracle.reduced_matmul(np.abs(H_g), np.abs(Wd_f), J),
                      kd)
    # against the oracle's whole block
    r = oracle.block.mlp_block(Xc, Wu_f, Wg_f, Wd_f, rho_up, rho_down)
    np.testing.assert_array_equal(I, r["I"])
    assert np.all(np.diff(J) > 0)
    diff = np.setxor1d(J, r["J"])
    thr = np.sort(r["ssH"])[::-1][kd - 1]
    assert np.all(np.abs(r["ssH"][diff] - thr) <= 1e-3 * thr), (diff, r["ssH"][diff], thr)
    if diff.size == 0:
        assert rel_fro(to_f64(Y), r["Y"]) <= 2e-3
    no_device_error()
