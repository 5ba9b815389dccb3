"""C-ABI library: loads, exports every symbol include/rmm.h declares, and its
host-side logic (k from rho, argument validation, workspace sizes) behaves —
no kernel launches, so these run without a GPU."""
import ctypes
import subprocess

import pytest

import oracle
import input_adaptive_reduced_score_b200 as R


def test_library_exports_every_declared_symbol():
    declared = R.declared_symbols()
    assert len(declared) >= 13
    missing = [s for s in declared if not hasattr(R.lib, s)]
    assert not missing, missing
    out = subprocess.run(["nm", "-D", "--defined-only", R.LIB_PATH], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(declared) <= exported
    # nothing beyond the ABI leaks out of the library
    assert {s for s in exported if s.startswith("rmm")} == set(declared)


def test_abi_version():
    assert R.rmm_abi_version() == 1


@pytest.mark.parametrize("rho,d", [(0.5, 4096), (0.7, 4096), (0.8, 4096), (1.0, 4096), (0.8, 14336),
                                   (0.8, 8192), (0.8, 28672), (0.5, 128), (0.3, 10), (1e-9, 100),
                                   (0.5, 1), (0.999, 7), (0.15, 7), (0.51, 100), (0.5, 32768)])
def test_k_from_rho_matches_oracle(rho, d):
    assert R.rmm_k_from_rho(rho, d) == oracle.k_from_rho(rho, d)


@pytest.mark.parametrize("rho", [0.0, -1.0, 1.5, float("nan")])
def test_k_from_rho_invalid(rho):
    assert R.rmm_k_from_rho(rho, 10) == -1


def _raw(name, *args):
    return getattr(R.lib, name)(*args)


def test_validation_rejects_before_launch():
    vp = ctypes.c_void_p
    s = vp(0)
    # null pointers / bad k / bad dtype are refused on the host
    assert _raw("rmm_topk", vp(0), 1, 10, 10, 3, vp(0), 3, s) == 1
    assert _raw("rmm_topk", vp(16), 1, 10, 10, 11, vp(16), 11, s) == 1
    assert _raw("rmm_topk", vp(16), 1, 10, 10, 0, vp(16), 3, s) == 1
    assert _raw("rmm_score", vp(16), 7, 1, 4, 4, 4, 0, vp(16), 4, 0, vp(0), 0, s) == 2
    assert _raw("rmm_score", vp(16), 1, 1, 4, 8, 4, 0, vp(16), 8, 0, vp(0), 0, s) == 1  # lda < d
    assert _raw("rmm_compact", vp(16), 1, 4, 8, 8, vp(16), 9, vp(16), 9, s) == 1       # k > d
    ws = vp(1 << 20)
    assert _raw("rmm_gemm", vp(16), 8, vp(16), 8, vp(16), 8, 4, 8, 0, 1, vp(16), 1, 8, ws, 1 << 20, s) == 1  # k = 0
    assert _raw("rmm_gemm", vp(16), 8, vp(16), 8, vp(16), 8, 4, 8, 4, 1, vp(16), 5, 8, ws, 1 << 20, s) == 2  # out dtype
    assert _raw("rmm_gemm", vp(18), 8, vp(16), 8, vp(16), 8, 4, 8, 4, 1, vp(16), 1, 8, ws, 1 << 20, s) == 2  # misaligned
    assert _raw("rmm_gemm", vp(16), 8, vp(16), 8, vp(16), 8, 4, 8, 4, 1, vp(16), 1, 8, vp(0), 0, s) == 3  # no workspace
    assert _raw("rmm_gather_rows", vp(16), 1, 0, 8, 8, vp(16), 4, vp(16), 8, s) == 1    # d = 0
    assert _raw("rmm_gather_rows", vp(16), 1, 8, 8, 12, vp(16), 4, vp(16), 12, s) == 2  # pitch not 16-byte
    assert _raw("rmm_compact_gather", vp(16), 8, vp(16), 8, 4, 8, 8, vp(0), 4, vp(16), 8, vp(16), 8, s) == 1  # null
    assert _raw("rmm_compact_gather", vp(16), 8, vp(16), 12, 4, 8, 12, vp(16), 4, vp(16), 8, vp(16), 16, s) == 2
    assert _raw("rmm_compact_gather", vp(16), 8, vp(16), 8, 4, 8, 8, vp(16), 9, vp(16), 9, vp(16), 8, s) == 1  # k > d
    assert _raw("rmm_matmul", vp(16), 8, vp(16), 8, 4, 8, 8, ctypes.c_double(1.5), 1, vp(16), 1, 8,
                vp(0), vp(0), vp(16), 1 << 20, s) == 1
    assert _raw("rmm_matmul", vp(16), 8, vp(16), 8, 4, 8, 8, ctypes.c_double(0.5), 1, vp(16), 1, 8,
                vp(0), vp(0), vp(0), 0, s) == 3  # workspace missing
    assert _raw("rmm_attention", vp(16), vp(16), vp(16), 1, 4, 3, 16, 64, ctypes.c_double(0.5),
                ctypes.c_double(0.5), ctypes.c_float(0), vp(16), 1, vp(0), vp(0), vp(0), vp(0), vp(16), 1 << 30,
                s) == 1  # Hq % Hkv
    assert _raw("rmm_attention", vp(16), vp(16), vp(16), 1, 4, 4, 16, 96, ctypes.c_double(0.5),
                ctypes.c_double(0.5), ctypes.c_float(0), vp(16), 1, vp(0), vp(0), vp(0), vp(0), vp(16), 1 << 30,
                s) == 2  # head_dim
    assert b"head_dim 96" in R.lib.rmm_last_error()


def test_validation_of_the_block_int8_decode_and_selftest_entry_points():
    """Each later entry point refuses bad arguments on the host, with the
    documented status, before any CUDA call (this runs without a GPU)."""
    vp, i64, dbl, flt = ctypes.c_void_p, ctypes.c_int64, ctypes.c_double, ctypes.c_float
    s, ws, big = vp(0), vp(1 << 20), 1 << 20
    INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 3
    # rmm_gemm_w8(A_I, ld_ai, Bq, ldb, b_scale, idx, d, M, N, k, Y, out_dtype, ldy, ws, ws_bytes, stream)
    assert _raw("rmm_gemm_w8", vp(16), 8, vp(16), 16, vp(16), vp(16), 8, 20, 8, 0, vp(16), 1, 8, ws, big, s) == INVALID
    assert _raw("rmm_gemm_w8", vp(16), 8, vp(16), 16, vp(16), vp(16), 8, 20, 8, 4, vp(16), 5, 8, ws, big, s) == UNSUPPORTED
    assert _raw("rmm_gemm_w8", vp(16), 8, vp(16), 16, vp(0), vp(16), 8, 20, 8, 4, vp(16), 1, 8, ws, big, s) == INVALID
    assert _raw("rmm_gemm_w8", vp(16), 8, vp(16), 24, vp(16), vp(16), 8, 20, 8, 4, vp(16), 1, 8, ws, big, s) == UNSUPPORTED
    assert _raw("rmm_gemm_w8", vp(16), 8, vp(16), 16, vp(16), vp(16), 8, 20, 8, 4, vp(16), 1, 8, vp(0), 0, s) == WORKSPACE
    # rmm_matmul_w8(A, lda, Bq, ldb, b_scale, M, d, N, rho, Y, out_dtype, ldy, idx_out, ss_out, ws, ws_bytes, stream)
    assert _raw("rmm_matmul_w8", vp(16), 8, vp(16), 16, vp(16), 20, 8, 8, dbl(1.5), vp(16), 1, 8, vp(0), vp(0), ws,
                big, s) == INVALID
    assert _raw("rmm_matmul_w8", vp(16), 8, vp(16), 24, vp(16), 20, 8, 8, dbl(0.5), vp(16), 1, 8, vp(0), vp(0), ws,
                big, s) == UNSUPPORTED
    assert _raw("rmm_matmul_w8", vp(16), 8, vp(16), 16, vp(16), 20, 8, 8, dbl(0.5), vp(16), 1, 8, vp(0), vp(0), vp(0),
                0, s) == WORKSPACE
    # rmm_matmul_multi(A, lda, M, d, rho, nprod, B[], ldb[], N[], Y[], ldy[], out_dtype, ss_in, idx_out, ss_out,
    #                  ws, ws_bytes, stream)
    Bs, Ys = (vp * 1)(16), (vp * 1)(16)
    Ns, ldys = (i64 * 1)(8), (i64 * 1)(8)
    ldb_ok, ldb_bad = (i64 * 1)(8), (i64 * 1)(12)
    args = lambda nprod, ldbs, w, wb: ("rmm_matmul_multi", vp(16), 8, 20, 8, dbl(0.5), nprod, Bs, ldbs, Ns, Ys, ldys,
                                       1, vp(0), vp(0), vp(0), w, wb, s)
    assert _raw(*args(0, ldb_ok, ws, big)) == INVALID
    assert _raw(*args(1, ldb_bad, ws, big)) == UNSUPPORTED
    assert _raw(*args(1, ldb_ok, vp(0), 0)) == WORKSPACE
    assert b"rmm_matmul_multi" in R.lib.rmm_last_error()
    # rmm_silu_mul_score(G, ldg, U, ldu, M, N, H, ldh, ss_out, ws, ws_bytes, stream)
    assert _raw("rmm_silu_mul_score", vp(16), 8, vp(16), 8, 4, 0, vp(16), 8, vp(16), ws, big, s) == INVALID
    assert _raw("rmm_silu_mul_score", vp(0), 8, vp(16), 8, 4, 8, vp(16), 8, vp(16), ws, big, s) == INVALID
    assert _raw("rmm_silu_mul_score", vp(16), 8, vp(20), 8, 4, 8, vp(16), 8, vp(16), ws, big, s) == UNSUPPORTED
    assert R.rmm_silu_mul_score_workspace_size(4096, 1024) > 0
    assert _raw("rmm_silu_mul_score", vp(16), 1024, vp(16), 1024, 4096, 1024, vp(16), 1024, vp(16), vp(0), 0,
                s) == WORKSPACE
    # rmm_mlp_block(X, ldx, M, d_model, d_ff, W_up, ld_up, W_gate, ld_gate, W_down, ld_down, rho_up, rho_down, Y,
    #               out_dtype, ldy, idx_up, idx_down, ws, ws_bytes, stream)
    mlp = lambda M, ru, w, wb: ("rmm_mlp_block", vp(16), 64, M, 64, 128, vp(16), 128, vp(16), 128, vp(16), 64,
                                dbl(ru), dbl(0.5), vp(16), 1, 64, vp(0), vp(0), w, wb, s)
    assert _raw(*mlp(0, 0.5, ws, big)) == INVALID
    assert _raw(*mlp(32, 0.0, ws, big)) == INVALID
    assert _raw(*mlp(32, 0.5, vp(0), 0)) == WORKSPACE
    # rmm_decode_attention(q, K, V, B, Hq, Hkv, L, Lmax, D, rho_d, rho_t, scale, O, out_dtype, idx_d, idx_t, lse,
    #                      logits, ws, ws_bytes, stream)
    dec = lambda Hq, Hkv, D, rt, q, out, w, wb: ("rmm_decode_attention", vp(q), vp(16), vp(16), 1, Hq, Hkv, 300, 300,
                                                 D, dbl(0.5), dbl(rt), flt(0), vp(16), out, vp(0), vp(0), vp(0),
                                                 vp(0), w, wb, s)
    assert _raw(*dec(8, 2, 128, 0.5, 16, 7, ws, big)) == UNSUPPORTED   # out dtype
    assert _raw(*dec(8, 3, 128, 0.5, 16, 1, ws, big)) == INVALID       # Hq % Hkv
    assert _raw(*dec(8, 2, 96, 0.5, 16, 1, ws, big)) == UNSUPPORTED    # head_dim
    assert _raw(*dec(6, 2, 128, 0.5, 16, 1, ws, big)) == UNSUPPORTED   # 3 q-heads per kv-head
    assert _raw(*dec(8, 2, 128, 0.0, 16, 1, ws, big)) == INVALID       # rho_t
    assert _raw(*dec(8, 2, 128, 0.5, 0, 1, ws, big)) == INVALID        # null q
    assert _raw(*dec(8, 2, 128, 0.5, 24, 1, ws, big)) == UNSUPPORTED   # misaligned q
    assert _raw(*dec(8, 2, 128, 0.5, 16, 1, vp(0), 0)) == WORKSPACE
    # rmm_selftest_timeout(which, stream)
    assert _raw("rmm_selftest_timeout", 3, s) == INVALID
    assert b"case 3" in R.lib.rmm_last_error()


def test_error_message_is_set():
    vp = ctypes.c_void_p
    assert R.lib.rmm_topk(vp(16), 1, 10, 10, 11, vp(16), 11, vp(0)) == 1
    assert b"k = 11" in R.lib.rmm_last_error()


def test_workspace_sizes():
    # one split needs no partial-sum workspace; many rows do
    assert R.rmm_score_workspace_size(1, 1, 8, 64) == 0
    big = R.rmm_score_workspace_size(1, 1, 4096, 4096)
    assert big > 0 and big % 256 == 0
    w = R.rmm_matmul_workspace_size(1, 4096, 4096, 14336, 0.5)
    # at least the compacted operands (M x k and k x N bf16) plus scores and indices
    assert w >= 4096 * 2048 * 2 + 2048 * 14336 * 2 + 4096 * 4 + 2048 * 4
    # B_I, then 2 + ceil(N / 256) counter words of the fused row copy (256-byte aligned)
    assert R.rmm_gemm_workspace_size(1, 14336, 2048) == 2048 * 14336 * 2 + 256
    assert R.rmm_gemm_workspace_size(1, 256 * 70, 64) == 64 * 256 * 70 * 2 + 512
    assert R.rmm_gemm_workspace_size(0, 128, 64) == 0
    assert R.rmm_matmul_workspace_size(1, 4096, 4096, 14336, 1.5) == 0


def test_workspace_sizes_of_the_later_entry_points():
    """Sizes cover the buffers each call carves from the workspace, are
    256-byte multiples, and are 0 for arguments the call would refuse."""
    M, d, N, rho = 4096, 4096, 14336, 0.5
    k = R.rmm_k_from_rho(rho, d)
    bi = k * N * 2
    # int8 weight: B_I is widened to bf16, so the same bytes as the bf16 product
    assert R.rmm_gemm_w8_workspace_size(N, k) == R.rmm_gemm_workspace_size(R.RMM_BF16, N, k)
    assert R.rmm_matmul_w8_workspace_size(M, d, N, rho) == R.rmm_matmul_workspace_size(R.RMM_BF16, M, d, N, rho)
    # shared selection: A_I plus the widest product's B_I (one product at a time)
    w = R.rmm_matmul_multi_workspace_size(M, d, N, rho)
    assert w >= M * k * 2 + bi and w % 256 == 0
    assert w == R.rmm_matmul_workspace_size(R.RMM_BF16, M, d, N, rho)
    assert R.rmm_matmul_multi_workspace_size(M, d, N, 0.0) == 0
    # gated MLP block: U, G and H (bf16 [M x d_ff]) and H's scores, plus the inner products' workspace
    dff = 14336
    wb = R.rmm_mlp_block_workspace_size(M, d, dff, 0.8, 0.5)
    inner = max(R.rmm_matmul_multi_workspace_size(M, d, dff, 0.8), R.rmm_matmul_multi_workspace_size(M, dff, d, 0.5))
    assert wb >= 3 * M * dff * 2 + dff * 4 + inner and wb % 256 == 0
    assert R.rmm_mlp_block_workspace_size(0, d, dff, 0.8, 0.5) == 0
    assert R.rmm_mlp_block_workspace_size(M, d, dff, 1.2, 0.5) == 0
    # SiLU * U with scores: partial sums only when rows are split
    assert R.rmm_silu_mul_score_workspace_size(4096, 1024) % 256 == 0
    assert R.rmm_silu_mul_score_workspace_size(4, 0) == 0
    # decode attention: the logits [B*Hq, L] and token indices [B*Hq, k_t] live in
    # the workspace unless the caller passes them
    B, Hq, L, D, rt = 2, 32, 32768, 128, 0.5
    kt = R.rmm_k_from_rho(rt, L)
    own = R.rmm_decode_attention_workspace_size(B, Hq, L, D, rt, False, False)
    given = R.rmm_decode_attention_workspace_size(B, Hq, L, D, rt, True, True)
    assert own >= given + B * Hq * L * 4 + B * Hq * kt * 4
    assert own % 256 == 0 and given % 256 == 0
