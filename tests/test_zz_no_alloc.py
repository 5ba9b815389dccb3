"""The allocation-free score entry point (rmm_score_noalloc).

Some callers cannot allocate device memory: a plugin handed only its input and
output buffers, or a process whose memory is reserved up front by an external
pool.  rmm_score_noalloc serves them by keeping the row-split partial sums of
the score in a fixed array inside the library.  Only inputs that the one-launch
kernel cannot read with 16-byte vectors use that array: fp32 activations and
bf16 whose base, row pitch or batch stride is not 16-byte aligned.  These
tests drive exactly those inputs through the C ABI (and the batched one through
the Python wrapper), two calls in a row each, and check that every call gives
bit for bit what rmm_score gives with a caller-provided workspace (same kernels,
same summation order) and agrees with the oracle's column norms.  One case sits
at the array's size limit; one just past it must be refused.  This file is
named to be collected last."""
import ctypes

import numpy as np
import pytest

import input_adaptive_reduced_score_b200 as R
import oracle
import workloads as W

LIMIT = 16 << 20  # RMM_SCORE_NOALLOC_MAX_BYTES in include/rmm.h


def test_oversized_call_is_refused():
    """Refused on the host, before any device work (runs without a GPU).
    fp32 always takes the partial-sum plan: 16385 x 16384 needs 257 row splits
    x 16384 columns x 4 B, just over the 16 MiB array."""
    b, M, d = 1, 16385, 16384
    assert R.rmm_score_workspace_size(R.RMM_F32, b, M, d) > LIMIT
    assert R.rmm_score_workspace_size(R.RMM_F32, b, M - 1, d) == LIMIT
    st = R.lib.rmm_score_noalloc(ctypes.c_void_p(256), R.RMM_F32, b, M, d, d, 0, ctypes.c_void_p(256), d, 0,
                                 ctypes.c_void_p(0))
    assert st == 1
    assert b"built-in" in R.lib.rmm_last_error()


def _noalloc_c(A, M, d, lda, out, dtype):
    import torch
    return R.lib.rmm_score_noalloc(ctypes.c_void_p(A.data_ptr()), dtype, 1, M, d, lda, 0,
                                   ctypes.c_void_p(out.data_ptr()), d, 0,
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _needs_workspace(A, dtype, b, M, d, lda, bstride):
    """rmm_score without a workspace is refused exactly when the call writes
    partial sums, i.e. when rmm_score_noalloc has to use its array."""
    import torch
    out = torch.empty((b, d), dtype=torch.float32, device="cuda")
    st = R.lib.rmm_score(ctypes.c_void_p(A.data_ptr()), dtype, b, M, d, lda, bstride, ctypes.c_void_p(out.data_ptr()),
                         d, 0, ctypes.c_void_p(0), 0, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st == 3  # RMM_ERR_WORKSPACE


@pytest.mark.gpu
@pytest.mark.parametrize("case", ["fp32", "bf16_odd_pitch", "bf16_at_limit", "bf16_aligned"])
def test_noalloc_matches_rmm_score_twice(case):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests.helpers import bf16_tensor
    if case == "fp32":
        bits = W.llm_activation_bf16(31, 4096, 4096)
        M, d = bits.shape
        A = torch.from_numpy(W.bf16_bits_to_f32(bits)).cuda()  # exact fp32 copies of the bf16 values
        dtype, lda = R.RMM_F32, d
        host = oracle.decode(bits, "bf16")
    elif case in ("bf16_odd_pitch", "bf16_at_limit"):
        # rows 3 elements (6 bytes) longer than d: the pitch is not a multiple of 16 bytes
        M, d = (3000, 14336) if case == "bf16_odd_pitch" else (16384, 16384)
        bits = W.llm_activation_bf16(32 if case == "bf16_odd_pitch" else 33, M, d)
        padded = np.zeros((M, d + 3), dtype=np.uint16)
        padded[:, :d] = bits
        A = bf16_tensor(padded)[:, :d]
        dtype, lda = R.RMM_BF16, d + 3
        host = oracle.decode(bits, "bf16") if case == "bf16_odd_pitch" else None
    else:
        bits = W.llm_activation_bf16(34, 4096, 4096)
        M, d = bits.shape
        A = bf16_tensor(bits)
        dtype, lda = R.RMM_BF16, d
        host = oracle.decode(bits, "bf16")
    uses_array = case != "bf16_aligned"
    assert _needs_workspace(A, dtype, 1, M, d, lda, 0) == uses_array
    if case == "bf16_at_limit":
        assert R.rmm_score_workspace_size(dtype, 1, M, d) == LIMIT   # the array's whole size
    ref = R.rmm_score(A)                                              # caller-provided workspace
    for _ in range(2):                                                # two calls in a row share the array
        out = torch.full((d,), -1.0, dtype=torch.float32, device="cuda")
        st = _noalloc_c(A, M, d, lda, out, dtype)
        assert st == 0, R.lib.rmm_last_error()
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    if host is None:  # at the limit: the oracle on a sample of columns
        cols = np.random.default_rng(7).choice(d, 512, replace=False)
        host_cols = oracle.decode(bits[:, cols], "bf16")
        np.testing.assert_allclose(out.cpu().numpy()[cols], oracle.column_sq_norms(host_cols), rtol=1e-5, atol=0)
    else:
        np.testing.assert_allclose(out.cpu().numpy(), oracle.column_sq_norms(host), rtol=1e-5, atol=0)
    assert R.rmm_device_error(clear=True) == 0


@pytest.mark.gpu
def test_noalloc_wrapper_batched_unaligned_stride():
    """Python wrapper, 3 matrices whose batch stride (M*d + 1 elements) is not
    16-byte aligned, so the batched partial-sum plan runs."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests.helpers import bf16_tensor
    b, M, d = 3, 1024, 4096
    mats = [W.llm_activation_bf16(40 + i, M, d) for i in range(b)]
    flat = np.zeros(b * (M * d + 1), dtype=np.uint16)
    for i, m in enumerate(mats):
        flat[i * (M * d + 1): i * (M * d + 1) + M * d] = m.ravel()
    A = bf16_tensor(flat).as_strided((b, M, d), (M * d + 1, d, 1))
    assert _needs_workspace(A, R.RMM_BF16, b, M, d, d, M * d + 1)
    ref = R.rmm_score(A)
    for _ in range(2):
        out = R.rmm_score_noalloc(A)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    got = out.cpu().numpy()
    for i, m in enumerate(mats):
        np.testing.assert_allclose(got[i], oracle.column_sq_norms(oracle.decode(m, "bf16")), rtol=1e-5, atol=0)
    assert R.rmm_device_error(clear=True) == 0
