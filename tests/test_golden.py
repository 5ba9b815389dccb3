"""The oracle still reproduces its committed golden fixture exactly."""
import json
import os

import numpy as np

import oracle
import workloads

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_tiny_fp32_golden():
    with open(os.path.join(HERE, "tiny_fp32_seed0.json")) as f:
        g = json.load(f)
    inp = workloads.tiny_fp32(0)
    A, B = oracle.decode(inp.A, "f32"), oracle.decode(inp.B, "f32")
    Y, idx, ss = oracle.rmm_path(A, B, 0.5)
    assert g["k"] == 128 == len(idx)
    assert list(idx) == g["idx"]
    np.testing.assert_array_equal(ss, [float.fromhex(h) for h in g["ss_hex"]])
    for r, row in zip(g["Y_rows"], g["Y_hex"]):
        np.testing.assert_allclose(Y[r], [float.fromhex(h) for h in row], rtol=1e-14, atol=0)
    assert abs(np.linalg.norm(Y) - float.fromhex(g["Y_fro_hex"])) <= 1e-12 * np.linalg.norm(Y)
