"""The allocation-free score entry point (rmm_score_noalloc).

Some callers cannot allocate device memory (a plugin handed only its input and
output buffers, a process whose memory is reserved up front by an external
pool).  rmm_score_noalloc serves them by keeping its partial sums in a fixed
array inside the library.  These tests call it through the C ABI and check
that two calls in a row give exactly what rmm_score gives with a
caller-provided workspace, and that shapes needing more scratch than the
array holds are refused.  This file is named to be collected last."""
import ctypes

import numpy as np
import pytest

import input_adaptive_reduced_score_b200 as R
import workloads as W

LIMIT = 16 << 20  # RMM_SCORE_NOALLOC_MAX_BYTES in include/rmm.h


def test_oversized_shape_is_refused():
    """Refused on the host, before any device work (runs without a GPU)."""
    # 4160 x 65536: 65 row splits x 65536 columns x 4 B = 17 MB of partial sums
    b, M, d = 1, 4160, 65536
    assert R.rmm_score_workspace_size(R.RMM_BF16, b, M, d) > LIMIT
    st = R.lib.rmm_score_noalloc(ctypes.c_void_p(256), R.RMM_BF16, b, M, d, d, 0, ctypes.c_void_p(256), d, 0,
                                 ctypes.c_void_p(0))
    assert st == 1
    assert b"built-in" in R.lib.rmm_last_error()


@pytest.mark.gpu
def test_noalloc_matches_rmm_score_twice():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tests.helpers import bf16_tensor
    cases = [W.llm_activation_bf16(31, 4096, 4096), W.llm_activation_bf16(32, 3000, 14336)]
    for bits in cases:
        M, d = bits.shape
        assert 0 < R.rmm_score_workspace_size(R.RMM_BF16, 1, M, d) <= LIMIT  # really uses the scratch
        A = bf16_tensor(bits)
        ref = R.rmm_score(A)                       # caller-provided workspace
        for _ in range(2):                         # two calls in a row share the scratch
            out = torch.full((d,), -1.0, dtype=torch.float32, device="cuda")
            st = R.lib.rmm_score_noalloc(ctypes.c_void_p(A.data_ptr()), R.RMM_BF16, 1, M, d, A.stride(0), 0,
                                         ctypes.c_void_p(out.data_ptr()), d, 0,
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
            assert st == 0, R.lib.rmm_last_error()
            torch.cuda.synchronize()
            np.testing.assert_allclose(out.cpu().numpy(), ref.cpu().numpy(), rtol=1e-5, atol=0)
    assert R.rmm_device_error(clear=True) == 0
