"""Input generator determinism and codec, and the score-gap conditioning."""
import numpy as np
import pytest

import workloads as W
from oracle import conditioning as C
from oracle import rmm as O


def test_bf16_codec_rne():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0, 1.0 + 2 ** -7], np.float32)
    bits = W.f32_to_bf16_bits(x)
    assert list(bits) == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x0000, 0x3F81]
    np.testing.assert_array_equal(W.bf16_bits_to_f64(bits), O.decode(bits, "bf16"))


def test_generator_is_deterministic_and_seeded():
    a = W.scaled_matmul_bf16(5, 64, 96, 40)
    b = W.scaled_matmul_bf16(5, 64, 96, 40)
    c = W.scaled_matmul_bf16(6, 64, 96, 40)
    assert np.array_equal(a.A, b.A) and np.array_equal(a.B, b.B)
    assert not np.array_equal(a.A, c.A)
    t = W.tiny_fp32(0)
    assert t.A.shape == (64, 256) and t.B.shape == (256, 128) and t.A.dtype == np.float32


def test_outlier_channels_count():
    X = W.bf16_bits_to_f64(W.llm_activation_bf16(1, 64, 4096))
    assert int(round(0.01 * 4096)) == 41
    assert X.shape == (64, 4096)


def test_attention_inputs_shapes():
    a = W.attention(seed=3, B=1, Hq=4, Hkv=2, S=32, D=16)
    assert a.Q.shape == (1, 4, 32, 16) and a.K.shape == (1, 2, 32, 16)
    b = W.attention(seed=3, B=1, Hq=4, Hkv=2, S=32, D=16, attempts=[0, 1])
    assert np.array_equal(a.Q[:, :2], b.Q[:, :2]) and not np.array_equal(a.Q[:, 2:], b.Q[:, 2:])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_gap_conditioning(dtype):
    if dtype == "bf16":
        A = W.scaled_matmul_bf16(3, 256, 512, 8, outlier_frac=0.0).A
    else:
        A = W.tiny_fp32(1).A
    d = A.shape[1]
    ks = [O.k_from_rho(r, d) for r in (0.5, 0.7, 0.8, 1.0)]
    A2, n = C.widen_topk_gaps(A, dtype, ks, rel_gap=2e-5)
    gaps, _ = C.boundary_gaps(O.column_sq_norms(O.decode(A2, dtype)), ks)
    assert all(g >= 2e-5 for g in gaps.values())
    changed = np.argwhere(A2 != A)
    assert len(changed) <= n
    if dtype == "bf16":
        diff = np.abs(A2.astype(np.int32) - A.astype(np.int32))
        assert diff.max() <= n  # each nudge moves one element by one ulp
    A3, n3 = C.widen_topk_gaps(A2, dtype, ks, rel_gap=2e-5)
    assert n3 == 0 and np.array_equal(A3, A2)
