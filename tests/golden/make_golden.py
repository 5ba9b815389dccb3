"""Writes the golden fixtures in this folder.  Calls only ``oracle`` and the
seeded generator ``workloads``; never the CUDA path.

The source page prints no worked numerical example, so the fixtures are the
oracle's own results on the seeded tiny fp32 workload, kept as a regression
lock on the oracle (any later change to its arithmetic must regenerate them and
say why).  Values are stored as fp64 hex strings so the text is exact.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import workloads  # noqa: E402


def tiny_case():
    inp = workloads.tiny_fp32(0)
    A = oracle.decode(inp.A, "f32")
    B = oracle.decode(inp.B, "f32")
    Y, idx, ss = oracle.rmm_path(A, B, 0.5)
    rows = [0, 17, 63]
    return {
        "workload": "reduced matmul fp32 64x256x128, seed 0, rho 0.5",
        "source": "Reduced Matrix Multiplication (technical summary), Metodologia: "
                  "Mecanismo Central, Estrategia de Seleccion",
        "k": int(len(idx)),
        "idx": [int(i) for i in idx],
        "ss_hex": [float(v).hex() for v in ss],
        "Y_rows": rows,
        "Y_hex": [[float(v).hex() for v in Y[r]] for r in rows],
        "Y_fro_hex": float(np.linalg.norm(Y)).hex(),
    }


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_fp32_seed0.json"), "w") as f:
        json.dump(tiny_case(), f, indent=0)
    print("wrote tiny_fp32_seed0.json")
