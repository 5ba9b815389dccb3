"""Writes attention_full_attempts.json: for each checked kv-group of the two
full-size attention workloads (32 heads x 8192 tokens; GQA 32/8 x 32768
tokens, head_dim 128, rho_d = rho_t = 0.5), the first redraw attempt of the
seeded generator whose every q-head has clear selection boundaries in the
fp64 oracle:

  head_dim:  (ss_(k) - ss_(k+1)) / ss_(k+1) >= 2e-5 at k_d = 64;
  tokens:    (t_(k) - t_(k+1)) / t_(k+1)    >= 1e-4 at k_t = S / 2,

with ss the column scores of Q and t_j = sum_{i>=j} P_ij^2 the token scores
(the reduced-attention readings of the method's summary, section Alcance de
Aplicación).  With those margins the fp32 scores the GPU computes cannot
order the boundary differently, so its index sets must equal the oracle's
bit for bit.  Only oracle/ and workloads/ are called.  A search takes tens of
minutes of CPU time; the test reads the stored attempts instead of searching.

    python tests/golden/make_attention_attempts.py [--procs 4]
"""
import argparse
import json
import multiprocessing as mp
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
OUT = os.path.join(HERE, "attention_full_attempts.json")

GAP_D = 2e-5
GAP_T = 1e-4
CONFIGS = {
    "attn_32h_8192": dict(seed=3, B=1, Hq=32, Hkv=32, S=8192, D=128, groups=[0, 11, 22, 31]),
    "attn_gqa32x8_32768": dict(seed=4, B=1, Hq=32, Hkv=8, S=32768, D=128, groups=[3]),
}


def evaluate(args):
    """Gaps of every q-head of kv-group g at one attempt (stops at the first
    head that misses a margin)."""
    name, g, attempt = args
    sys.path.insert(0, ROOT)
    import numpy as np

    import oracle
    import workloads as W
    from oracle import attention as OA
    from oracle.conditioning import boundary_gaps
    c = CONFIGS[name]
    S, D, G = c["S"], c["D"], c["Hq"] // c["Hkv"]
    kd, kt = oracle.k_from_rho(0.5, D), oracle.k_from_rho(0.5, S)
    Qg, Kg, _ = W.attention_group(c["seed"], c["B"], c["Hq"], c["Hkv"], S, D, g, attempt)
    K = oracle.decode(W.f32_to_bf16_bits(Kg[0]), "bf16")
    gaps = []
    for q in range(G):
        Q = oracle.decode(W.f32_to_bf16_bits(Qg[0, q]), "bf16")
        gd = boundary_gaps(oracle.column_sq_norms(Q), [kd])[0][kd]
        if gd < GAP_D:
            return name, g, attempt, False, gaps + [(float(gd), None)]
        sel = OA.head_dim_selection(Q, 0.5)
        L = OA.lse_rows(Q, K, sel, np.arange(S))
        t = OA.token_scores(Q, K, sel, L, np.arange(S))
        gt = boundary_gaps(t, [kt])[0][kt]
        gaps.append((float(gd), float(gt)))
        if gt < GAP_T:
            return name, g, attempt, False, gaps
    return name, g, attempt, True, gaps


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--procs", type=int, default=4)
    ap.add_argument("--max-attempts", type=int, default=200)
    a = ap.parse_args()
    os.environ.setdefault("OPENBLAS_NUM_THREADS", "2")
    result = {"gap_head_dim": GAP_D, "gap_tokens": GAP_T, "configs": {}}
    ctx = mp.get_context("spawn")
    with ctx.Pool(a.procs) as pool:
        for name, c in CONFIGS.items():
            entry = {k: v for k, v in c.items() if k != "groups"}
            entry["attempts"] = {}
            entry["gaps"] = {}
            for g in c["groups"]:
                found = None
                for base in range(0, a.max_attempts, a.procs):
                    outs = pool.map(evaluate, [(name, g, base + i) for i in range(a.procs)])
                    for _, _, att, ok, gaps in sorted(outs, key=lambda o: o[2]):
                        print(f"{name} group {g} attempt {att}: {'ok' if ok else 'no'} {gaps}", flush=True)
                        if ok and found is None:
                            found = (att, gaps)
                    if found:
                        break
                if not found:
                    raise SystemExit(f"{name} group {g}: no attempt below {a.max_attempts} has clear margins")
                entry["attempts"][str(g)] = found[0]
                entry["gaps"][str(g)] = found[1]
            result["configs"][name] = entry
    with open(OUT, "w") as f:
        json.dump(result, f, indent=1)
    print("wrote", OUT)


if __name__ == "__main__":
    main()
