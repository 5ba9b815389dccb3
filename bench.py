#!/usr/bin/env python
"""Benchmark of the reduced-matrix-multiplication hot path on B200.

One step = the whole path on one batch of the MLP up/gate projection
workload (X [4096 x 4096] bf16 activation with per-channel lognormal scale
and 1% outlier channels, W [4096 x 14336] bf16 ~ N(0, 0.02^2), rho = 0.5):
column scores -> top-k -> compaction of X -> tcgen05 reduced GEMM whose
spare warps gather the kept rows of W while it multiplies, every stage a
librmm kernel called through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl rmm|reference]

Prints one JSON line (rank 0).  `value` is the effective throughput
2*M*N*k / step time in TFLOP/s over all ranks (weak scaling: each rank runs
its own batch, no data-path collective).  Timing: K steps between a barrier
and a device synchronisation; each step is bracketed by CUDA events on the
launching stream and the step times are summed; a 256 MiB buffer is written
between steps (L2 flush) outside the event intervals; the max over ranks is
reported.  `--impl reference` times the fp64 CPU oracle on a bounded sample of
the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import faulthandler
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)
faulthandler.enable()

METRIC = "reduced-GEMM effective TFLOP/s & speedup vs dense bf16 at rho=0.5; % roofline"
WORKLOAD = "MLP up/gate projection: X[4096x4096] bf16 (lognormal channel scale, 1% outliers x20) · W[4096x14336] bf16 N(0,0.02^2), rho=0.5"
M, D, N, RHO = 4096, 4096, 14336, 0.5
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
GEMM_SOURCES = ["input_adaptive_reduced_score_b200/csrc/rmm_gemm_tc.cu",
                "input_adaptive_reduced_score_b200/csrc/rmm_launch.cuh",
                "input_adaptive_reduced_score_b200/csrc/rmm_device.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "rmm_gemm_tc_mlp_up_traffic.json")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["rmm", "reference"], default="rmm")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", choices=["bench", "matmul", "attention", "attention_gqa", "layer70b", "decode", "w8",
                                       "decode_attention", "block", "down", "topk"],
                    default="bench",
                    help="matmul / attention / attention_gqa / layer70b / decode / w8 / decode_attention / block / "
                         "down / topk: run only that workload a few "
                         "times and exit (a short program for profiler captures; prints no JSON line)")
    a = ap.parse_args()
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    return a


def k_of(rho, d):
    import math
    return min(max(math.ceil(rho * d - 1e-9 * d), 1), d)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return {k: float(j[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def sources_sha(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def traffic_per_launch():
    """DRAM bytes per GEMM launch from the committed ncu capture, or None when
    the kernel sources changed since it was taken."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        if t.get("sources_sha256") != sources_sha(GEMM_SOURCES):
            return None
        return float(t["dram_bytes_per_launch"])
    except Exception:
        return None


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read-only)."""
    NAMES = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
             0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
             0x1: "gpu_idle"}

    @staticmethod
    def _handle(nv, props):
        """NVML handle of the torch device: by UUID, else by a formatted PCI bus id string."""
        uuid = str(getattr(props, "uuid", "") or "")
        if uuid:
            try:
                return nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                pass
        bus_id = f"{int(props.pci_domain_id):08x}:{int(props.pci_bus_id):02x}:{int(props.pci_device_id):02x}.0"
        return nv.nvmlDeviceGetHandleByPciBusId(bus_id)

    def __init__(self, props):
        self.samples, self.reasons, self.max_mhz, self.err = [], 0, None, None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = self._handle(pynvml, props)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - reported, not fatal
            self.nv, self.err = None, repr(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                fn = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
                self.reasons |= fn(self.h)
            except Exception as e:
                self.err = repr(e)
            time.sleep(0.01)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.nv:
            self.t.join()

    def summary(self):
        names = sorted(n for bit, n in self.NAMES.items() if self.reasons & bit)
        med = statistics.median(self.samples) if self.samples else None
        out = {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}
        if self.err:
            out["error"] = self.err
        return out

    def rejected(self):
        s = self.summary()
        bad = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"} & set(s["reasons"])
        stuck = (s["sm_mhz"] is not None and self.max_mhz and s["sm_mhz"] < 0.5 * self.max_mhz
                 and not s["reasons"])
        return bool(bad) or bool(stuck)


# ------------------------------------------------------------------ CPU oracle timing

def bench_config(world):
    """The workload's config, identical in both arms' JSON lines."""
    return {"workload": WORKLOAD, "M": M, "d": D, "N": N, "rho": RHO, "k": k_of(RHO, D),
            "l2": "256 MiB buffer written between steps, outside the timed intervals",
            "parallelism": f"independent batch per GPU x{world}"}


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_sample_step(oracle, Xf, Wf, rows, k):
    """One bounded sample of the workload through the fp64 oracle: scores and
    top-k over the sampled rows' activation, reduced product of those rows."""
    A = Xf[rows]
    ss = oracle.column_sq_norms(A)
    idx = oracle.topk_indices(ss, k)
    Y = oracle.reduced_matmul(A, Wf, idx)
    return Y


def cpu_oracle_inputs():
    import workloads
    import oracle
    X = workloads.llm_activation_bf16(1, M, D)
    Wb = workloads.weight_bf16(1, D, N)
    return oracle, oracle.decode(X, "bf16"), oracle.decode(Wb, "bf16")


def time_cpu_oracle(target_s=15.0):
    """CPU baseline: the oracle as it stands on the host cores; the row count
    of the sample is sized to about `target_s` seconds of work."""
    oracle, Xf, Wf = cpu_oracle_inputs()
    k = k_of(RHO, D)
    t0 = time.perf_counter()
    oracle_sample_step(oracle, Xf, Wf, list(range(32)), k)
    t32 = time.perf_counter() - t0
    rows_n = int(max(32, min(M, 32 * target_s / max(t32, 1e-3))) // 32 * 32)
    rows = list(range(rows_n))
    t0 = time.perf_counter()
    oracle_sample_step(oracle, Xf, Wf, rows, k)
    t = time.perf_counter() - t0
    tflops = 2.0 * rows_n * N * k / t / 1e12
    return {"value": tflops, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"fp64 oracle on the first {rows_n} of {M} rows (scores, top-k and reduced product of "
                      f"the sampled rows), {t:.1f} s"}


def run_reference(args):
    """Reference arm: the fp64 CPU oracle, timed step by step on bounded samples."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    oracle, Xf, Wf = cpu_oracle_inputs()
    k = k_of(RHO, D)
    t0 = time.perf_counter()
    oracle_sample_step(oracle, Xf, Wf, list(range(16)), k)
    t16 = time.perf_counter() - t0
    budget = 150.0 / (args.steps + args.warmup)
    rows_n = int(max(8, min(M, 16 * budget / max(t16, 1e-3))) // 8 * 8)
    for i in range(args.warmup):
        oracle_sample_step(oracle, Xf, Wf, list(range(rows_n)), k)
    t0 = time.perf_counter()
    for i in range(args.steps):
        r0 = (i * rows_n) % (M - rows_n + 1)
        oracle_sample_step(oracle, Xf, Wf, list(range(r0, r0 + rows_n)), k)
    t = time.perf_counter() - t0
    value = 2.0 * rows_n * N * k * args.steps / t / 1e12
    cores = cpu_threads()
    sample = (f"each step: fp64 oracle on {rows_n} of {M} rows (scores, top-k, reduced product), on the host "
              "cores; no GPU and so no L2 flush; value scaled to the FLOPs of the rows processed")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": bench_config(args.gpus),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm

def aggregate(local_ms, local_flops, world):
    """Max of step-time totals and sum of flops over ranks (no-op at world 1)."""
    import torch
    if world == 1:
        return local_ms, local_flops
    import torch.distributed as dist
    t = torch.tensor([local_ms], dtype=torch.float64)
    f = torch.tensor([local_flops], dtype=torch.float64)
    if dist.get_backend() == "nccl":
        t, f = t.cuda(), f.cuda()
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(f, op=dist.ReduceOp.SUM)
    return float(t.item()), float(f.item())


ATTN = dict(B=1, Hq=32, Hkv=32, S=8192, D=128, rho_d=0.5, rho_t=0.5, seed=3)
ATTN_GQA = dict(B=1, Hq=32, Hkv=8, S=32768, D=128, rho_d=0.5, rho_t=0.5, seed=4)
EX2_PER_CLK_SM = 16  # exp unit (MUFU ex2) results per clock per SM, measured with a throughput probe


def measure_attention(R, workloads, bf16_tensor, dev, stream, flush, steps, timed, peaks, a=ATTN):
    """Reduced attention (same flush and event protocol as the GEMM path), next
    to torch's causal SDPA (flash/cuDNN; for GQA the kv heads are repeated
    once, outside the timed region).  Rooflines of the whole pipeline: the
    tensor-core work (logits of passes A and B over the causal pairs at k_d,
    logits and P V of pass C over the kept causal pairs) at the measured bf16
    peak, and the exponentials (one per causal pair in each of passes A and
    B, one per kept causal pair in pass C) at 16 per clock per SM at the SM
    clock sampled during the timed calls."""
    import numpy as np
    import torch
    inp = workloads.attention(a["seed"], a["B"], a["Hq"], a["Hkv"], a["S"], a["D"], a["rho_d"], a["rho_t"])
    Q, K, V = (bf16_tensor(x, dev) for x in (inp.Q, inp.K, inp.V))
    del inp
    O = torch.empty_like(Q)
    B, Hq, Hkv, S, D = a["B"], a["Hq"], a["Hkv"], a["S"], a["D"]
    kd, kt = R.rmm_k_from_rho(a["rho_d"], D), R.rmm_k_from_rho(a["rho_t"], S)
    idx_t = torch.empty((B * Hq, kt), dtype=torch.int32, device=dev)
    ws = torch.empty(R.rmm_attention_workspace_size(B, Hq, Hkv, S, D, a["rho_d"], a["rho_t"]), dtype=torch.uint8,
                     device=dev)
    Kr = K if Hkv == Hq else K.repeat_interleave(Hq // Hkv, 1)
    Vr = V if Hkv == Hq else V.repeat_interleave(Hq // Hkv, 1)

    def rmm(ev):
        ev[0].record(stream)
        R.rmm_attention(Q, K, V, a["rho_d"], a["rho_t"], out=O, idx_t=idx_t, ws=ws)
        ev[1].record(stream)

    def sdpa(ev):
        ev[0].record(stream)
        torch.nn.functional.scaled_dot_product_attention(Q, Kr, Vr, is_causal=True)
        ev[1].record(stream)

    for fn in (rmm, sdpa):
        for _ in range(3):
            fn([torch.cuda.Event(enable_timing=True) for _ in range(2)])
    with ClockSampler(torch.cuda.get_device_properties(dev)) as clk:
        rmm_ms = statistics.mean(p[0] for p in timed(rmm, steps, 2))
    sdpa_ms = statistics.mean(p[0] for p in timed(sdpa, steps, 2))
    if R.rmm_device_error(stream) != 0:
        raise SystemExit("device error during the attention runs")
    H = B * Hq
    pairs = H * S * (S + 1) / 2.0
    pos = idx_t.cpu().numpy().astype(np.int64)
    kept_pairs = float(np.sum(S - pos))           # queries i >= pos_r, summed over kept tokens and heads
    flops = 2.0 * kd * pairs * 2 + 2.0 * (kd + D) * kept_pairs
    exps = 2.0 * pairs + kept_pairs
    ck = clk.summary()
    mhz = ck["sm_mhz"] or 1965.0
    tensor_floor_ms = flops / (peaks["bf16_tflops"] * 1e12) * 1e3
    exp_floor_ms = exps / (EX2_PER_CLK_SM * 148 * mhz * 1e6) * 1e3
    dense_flops = 4.0 * (S * (S + 1) / 2) * D * H
    return {"workload": f"causal attention B{B} Hq{Hq} Hkv{Hkv} S{S} D{D}, rho_d={a['rho_d']} rho_t={a['rho_t']}, "
                        "Q/K/V N(0,1) x per-dim lognormal(0,0.5)",
            "ms": rmm_ms, "sdpa_ms": sdpa_ms, "speedup_vs_sdpa": sdpa_ms / rmm_ms,
            "dense_equivalent_tflops": dense_flops / (rmm_ms * 1e-3) / 1e12,
            "sdpa_tflops": dense_flops / (sdpa_ms * 1e-3) / 1e12,
            "kept_pair_frac": kept_pairs / pairs,
            "roofline": {"tensor": {"flops": flops, "floor_ms": tensor_floor_ms, "frac": tensor_floor_ms / rmm_ms,
                                    "peak_tflops": peaks["bf16_tflops"]},
                         "exp_unit": {"exps": exps, "floor_ms": exp_floor_ms, "frac": exp_floor_ms / rmm_ms,
                                      "ex2_per_clk_sm": EX2_PER_CLK_SM, "sm_mhz": mhz},
                         "bound": "exp_unit" if exp_floor_ms > tensor_floor_ms else "tensor"},
            "clocks": ck, "gpu_launches_per_call": 12, "calls": steps}


def measure_layer70b(R, workloads, bf16_tensor, dev, stream, flush, steps, timed, peaks):
    """The 70B-shaped layer (2048 tokens, hidden 8192, MLP 28672; q/k/v/o at
    rho = 0.5, up/gate/down at rho = 0.8), each projection on its own drawn
    activation: the rmm_matmul step, the selection alone (score + top-k, one
    event interval), the product alone (rmm_gemm on the compacted activation,
    an event before and after it) and cuBLAS on the same shape, all with a
    256 MiB write between calls.  q, k and v also run as one rmm_matmul_multi
    call on q's activation (one selection for the three weights)."""
    import torch
    out = {}
    qkv = {}
    for name, Mg, dg, Ng, rho in workloads.layer70b_gemms():
        inp = workloads.layer70b_inputs(name)
        X, Wt = bf16_tensor(inp.A, dev), bf16_tensor(inp.B, dev)
        del inp
        k = R.rmm_k_from_rho(rho, dg)
        Y = torch.empty((Mg, Ng), dtype=torch.bfloat16, device=dev)
        ss = torch.empty(dg, dtype=torch.float32, device=dev)
        idx = torch.empty(k, dtype=torch.int32, device=dev)
        AI = torch.empty((Mg, (k + 7) // 8 * 8), dtype=torch.bfloat16, device=dev)[:, :k]
        mws = torch.empty(R.rmm_matmul_workspace_size(R.RMM_BF16, Mg, dg, Ng, rho), dtype=torch.uint8, device=dev)
        gws = torch.empty(R.rmm_gemm_workspace_size(R.RMM_BF16, Ng, k), dtype=torch.uint8, device=dev)
        sws = torch.empty(max(R.rmm_score_workspace_size(R.RMM_BF16, 1, Mg, dg), 256), dtype=torch.uint8, device=dev)

        def step(ev):
            ev[0].record(stream)
            R.rmm_matmul(X, Wt, rho, out=Y, ws=mws)
            ev[1].record(stream)

        def split(ev):
            ev[0].record(stream)
            R.rmm_score(X, out=ss, ws=sws)
            R.rmm_topk(ss, k, out=idx)
            ev[1].record(stream)
            R.rmm_compact(X, idx, out=AI)
            ev[2].record(stream)
            R.rmm_gemm(AI, Wt, idx, out=Y, ws=gws)
            ev[3].record(stream)

        def dense(ev):
            ev[0].record(stream)
            torch.matmul(X, Wt, out=Y)
            ev[1].record(stream)
        for _ in range(3):
            step([torch.cuda.Event(enable_timing=True) for _ in range(2)])
            split([torch.cuda.Event(enable_timing=True) for _ in range(4)])
            dense([torch.cuda.Event(enable_timing=True) for _ in range(2)])
        ms = statistics.mean(p[0] for p in timed(step, steps, 2))
        sp = timed(split, steps, 4)
        sel_ms = statistics.mean(p[0] for p in sp)
        gemm_ms = statistics.mean(p[2] for p in sp)
        dms = statistics.mean(p[0] for p in timed(dense, steps, 2))
        if R.rmm_device_error(stream) != 0:
            raise SystemExit(f"device error during the 70B-layer {name} runs")
        fl = 2.0 * Mg * Ng * k
        out[name] = {"M": Mg, "d": dg, "N": Ng, "rho": rho, "k": k, "step_us": ms * 1e3,
                     "effective_tflops": fl / (ms * 1e-3) / 1e12, "dense_us": dms * 1e3,
                     "speedup_vs_dense": dms / ms, "select_us": sel_ms * 1e3,
                     "select_frac_of_dense": sel_ms / dms, "gemm_us": gemm_ms * 1e3,
                     "gemm_roofline_frac": fl / (gemm_ms * 1e-3) / 1e12 / peaks["bf16_tflops"]}
        if name == "q_proj":
            qkv["X"], qkv["q"] = X, Wt
        elif name in ("k_proj", "v_proj"):
            qkv[name[0]] = Wt
        del Y, AI, mws, gws
    # q, k, v on one activation: one selection, three products
    X, Ws = qkv["X"], [qkv["q"], qkv["k"], qkv["v"]]
    Ys = [torch.empty((X.shape[0], w.shape[1]), dtype=torch.bfloat16, device=dev) for w in Ws]
    ws = torch.empty(R.rmm_matmul_multi_workspace_size(X.shape[0], X.shape[1], max(w.shape[1] for w in Ws), 0.5),
                     dtype=torch.uint8, device=dev)

    def multi(ev):
        ev[0].record(stream)
        R.rmm_matmul_multi(X, Ws, 0.5, outs=Ys, ws=ws)
        ev[1].record(stream)

    def dense3(ev):
        ev[0].record(stream)
        for w, y in zip(Ws, Ys):
            torch.matmul(X, w, out=y)
        ev[1].record(stream)
    for _ in range(3):
        multi([torch.cuda.Event(enable_timing=True) for _ in range(2)])
        dense3([torch.cuda.Event(enable_timing=True) for _ in range(2)])
    ms = statistics.mean(p[0] for p in timed(multi, steps, 2))
    dms = statistics.mean(p[0] for p in timed(dense3, steps, 2))
    if R.rmm_device_error(stream) != 0:
        raise SystemExit("device error during the 70B-layer q/k/v runs")
    k = R.rmm_k_from_rho(0.5, X.shape[1])
    fl = sum(2.0 * X.shape[0] * w.shape[1] * k for w in Ws)
    out["qkv_shared_selection"] = {"step_us": ms * 1e3, "dense_us": dms * 1e3, "speedup_vs_dense": dms / ms,
                                   "effective_tflops": fl / (ms * 1e-3) / 1e12}
    tot = sum(v["step_us"] for n, v in out.items() if n.endswith("_proj"))
    tot_dense = sum(v["dense_us"] for n, v in out.items() if n.endswith("_proj"))
    out["layer_total"] = {"step_us": tot, "dense_us": tot_dense, "speedup_vs_dense": tot_dense / tot}
    out["workload"] = ("70B-shaped layer: 2048 tokens, hidden 8192, MLP 28672; activations as the MLP up "
                       "projection's (lognormal channel scale, 1% outliers x20), weights N(0, 0.02^2)")
    return out


def measure_decode(R, workloads, bf16_tensor, dev, stream, flush, steps, timed, Wt, hbm_gbs):
    """Decode-sized products (M = 1 and 16 activation rows) on the MLP up/gate
    weight through rmm_matmul (one selection launch: scores, top-k and A_I;
    then the row-streaming product that reads only the kept rows of W), next
    to cuBLAS on the full W (same flush protocol).  The product is also timed
    alone; its bandwidth counts its algorithmic bytes: the k kept rows of W,
    A_I and Y."""
    import torch
    out = {}
    for rows in (1, 16):
        X = bf16_tensor(workloads.llm_activation_bf16(7 + rows, rows, D), dev)
        k = R.rmm_k_from_rho(RHO, D)
        ss = torch.empty(D, dtype=torch.float32, device=dev)
        idx = torch.empty(k, dtype=torch.int32, device=dev)
        AI = torch.empty((rows, (k + 7) // 8 * 8), dtype=torch.bfloat16, device=dev)[:, :k]
        Y = torch.empty((rows, N), dtype=torch.bfloat16, device=dev)
        Yd = torch.empty_like(Y)
        sws = torch.empty(max(256, R.rmm_score_workspace_size(R.RMM_BF16, 1, rows, D)), dtype=torch.uint8, device=dev)
        gws = torch.empty(R.rmm_gemm_workspace_size(R.RMM_BF16, N, k), dtype=torch.uint8, device=dev)

        mws = torch.empty(R.rmm_matmul_workspace_size(R.RMM_BF16, rows, D, N, RHO), dtype=torch.uint8, device=dev)

        def rmm(ev):
            # the whole path as a user calls it: one selection launch, then the product
            ev[0].record(stream)
            R.rmm_matmul(X, Wt, RHO, out=Y, idx_out=idx, ws=mws)
            ev[1].record(stream)

        def product(ev):
            ev[0].record(stream)
            R.rmm_gemm(AI, Wt, idx, out=Y, ws=gws)
            ev[1].record(stream)

        def dense(ev):
            ev[0].record(stream)
            torch.matmul(X, Wt, out=Yd)
            ev[1].record(stream)

        for _ in range(3):
            rmm([torch.cuda.Event(enable_timing=True) for _ in range(2)])
            dense([torch.cuda.Event(enable_timing=True) for _ in range(2)])
        R.rmm_compact(X, idx, out=AI)
        for _ in range(3):
            product([torch.cuda.Event(enable_timing=True) for _ in range(2)])
        step_ms = statistics.mean(p[0] for p in timed(rmm, steps, 2))
        prod_ms = statistics.mean(p[0] for p in timed(product, steps, 2))
        dense_ms = statistics.mean(p[0] for p in timed(dense, steps, 2))
        prod_bytes = 2.0 * k * N + 2.0 * rows * k + 2.0 * rows * N
        gbs = prod_bytes / (prod_ms * 1e-3) / 1e9
        out[f"M{rows}"] = {"step_us": step_ms * 1e3, "product_us": prod_ms * 1e3, "product_GB/s": gbs,
                           "product_frac_hbm": gbs / hbm_gbs, "dense_us": dense_ms * 1e3,
                           "speedup_vs_dense": dense_ms / step_ms}
    if R.rmm_device_error(stream) != 0:
        raise SystemExit("device error during the decode runs")
    out["workload"] = (f"decode rows x[1 or 16 x {D}] (lognormal channel scale, outliers) . W[{D}x{N}], rho={RHO}; "
                       "W streamed from HBM (256 MiB flush between steps)")
    return out


def measure_w8(R, workloads, bf16_tensor, dev, stream, flush, steps, timed, X, hbm_gbs):
    """The same products with an int8 weight (per-column fp32 scales):
    rmm_matmul_w8 on the MLP up/gate activation (selection, one launch that
    compacts A and widens the kept int8 rows to bf16, the tensor-core product
    with the scales in its epilogue), and the decode product on 1 and 16 rows
    (kept int8 rows read in place).  Product bandwidth counts its algorithmic
    bytes: k kept int8 rows, the scales, A_I and Y."""
    import torch
    q, sc = workloads.weight_int8(1, D, N)
    Wq = torch.from_numpy(q).to(dev)
    S = torch.from_numpy(sc).to(dev)
    k = R.rmm_k_from_rho(RHO, D)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    mws = torch.empty(R.rmm_matmul_w8_workspace_size(M, D, N, RHO), dtype=torch.uint8, device=dev)

    def path(ev):
        ev[0].record(stream)
        R.rmm_matmul_w8(X, Wq, S, RHO, out=Y, ws=mws)
        ev[1].record(stream)
    for _ in range(3):
        path([torch.cuda.Event(enable_timing=True) for _ in range(2)])
    ms = statistics.mean(p[0] for p in timed(path, steps, 2))
    out = {"prefill": {"ms": ms, "effective_tflops": 2.0 * M * N * k / (ms * 1e-3) / 1e12,
                       "gpu_launches_per_call": 4}}
    gws = torch.empty(R.rmm_gemm_w8_workspace_size(N, k), dtype=torch.uint8, device=dev)
    for rows in (1, 16):
        Xr = bf16_tensor(workloads.llm_activation_bf16(7 + rows, rows, D), dev)
        idx = torch.empty(k, dtype=torch.int32, device=dev)
        Yr = torch.empty((rows, N), dtype=torch.bfloat16, device=dev)
        rws = torch.empty(R.rmm_matmul_w8_workspace_size(rows, D, N, RHO), dtype=torch.uint8, device=dev)

        def step(ev):
            ev[0].record(stream)
            R.rmm_matmul_w8(Xr, Wq, S, RHO, out=Yr, idx_out=idx, ws=rws)
            ev[1].record(stream)
        for _ in range(3):
            step([torch.cuda.Event(enable_timing=True) for _ in range(2)])
        AI = R.rmm_compact(Xr, idx)

        def product(ev):
            ev[0].record(stream)
            R.rmm_gemm_w8(AI, Wq, S, idx, out=Yr, ws=gws)
            ev[1].record(stream)
        for _ in range(3):
            product([torch.cuda.Event(enable_timing=True) for _ in range(2)])
        step_ms = statistics.mean(p[0] for p in timed(step, steps, 2))
        prod_ms = statistics.mean(p[0] for p in timed(product, steps, 2))
        prod_bytes = 1.0 * k * N + 4.0 * N + 2.0 * rows * k + 2.0 * rows * N
        gbs = prod_bytes / (prod_ms * 1e-3) / 1e9
        out[f"M{rows}"] = {"step_us": step_ms * 1e3, "product_us": prod_ms * 1e3, "product_GB/s": gbs,
                           "product_frac_hbm": gbs / hbm_gbs}
    if R.rmm_device_error(stream) != 0:
        raise SystemExit("device error during the int8-weight runs")
    out["workload"] = (f"X[{M} or 1 or 16 x {D}] bf16 . W[{D}x{N}] int8 with per-column fp32 scales "
                       f"(symmetric absmax storage of N(0, 0.02^2)), rho={RHO}; 256 MiB flush between steps")
    return out


def measure_block(R, workloads, bf16_tensor, dev, stream, flush, steps, timed, X):
    """The block driver on the MLP up/gate activation X [4096 x 4096]:
    (1) q/k/v-shaped products (W 4096 x 4096, 4096 x 1024, 4096 x 1024) at
    rho = 0.5 with one shared selection (rmm_matmul_multi) against three
    rmm_matmul calls; (2) the gated MLP block (d_ff = 14336, rho_up = 0.8,
    rho_down = 0.5; up/gate share one selection, the down projection's scores
    come from the fused SiLU * U producer) against the same chain built from
    rmm_matmul calls and a torch SiLU * U, and against dense cuBLAS."""
    import torch
    out = {}
    Ws = [bf16_tensor(workloads.weight_bf16(9, D, n, group=i), dev) for i, n in enumerate((D, 1024, 1024))]
    Ys = [torch.empty((M, w.shape[1]), dtype=torch.bfloat16, device=dev) for w in Ws]
    mws = torch.empty(R.rmm_matmul_multi_workspace_size(M, D, D, 0.5), dtype=torch.uint8, device=dev)
    sws = [torch.empty(R.rmm_matmul_workspace_size(R.RMM_BF16, M, D, w.shape[1], 0.5), dtype=torch.uint8, device=dev)
           for w in Ws]

    def shared(ev):
        ev[0].record(stream)
        R.rmm_matmul_multi(X, Ws, 0.5, outs=Ys, ws=mws)
        ev[1].record(stream)

    def separate(ev):
        ev[0].record(stream)
        for w, y, ws_ in zip(Ws, Ys, sws):
            R.rmm_matmul(X, w, 0.5, out=y, ws=ws_)
        ev[1].record(stream)
    for _ in range(3):
        shared([torch.cuda.Event(enable_timing=True) for _ in range(2)])
        separate([torch.cuda.Event(enable_timing=True) for _ in range(2)])
    out["qkv_shared_selection"] = {"shared_us": statistics.mean(p[0] for p in timed(shared, steps, 2)) * 1e3,
                                   "separate_us": statistics.mean(p[0] for p in timed(separate, steps, 2)) * 1e3}
    del Ws, Ys, mws, sws
    F = 14336
    Wu = bf16_tensor(workloads.weight_bf16(10, D, F, group=0), dev)
    Wg = bf16_tensor(workloads.weight_bf16(10, D, F, group=1), dev)
    Wd = bf16_tensor(workloads.weight_bf16(10, F, D, group=2), dev)
    Y = torch.empty((M, D), dtype=torch.bfloat16, device=dev)
    bws = torch.empty(R.rmm_mlp_block_workspace_size(M, D, F, 0.8, 0.5), dtype=torch.uint8, device=dev)
    U = torch.empty((M, F), dtype=torch.bfloat16, device=dev)
    G = torch.empty_like(U)
    uws = torch.empty(R.rmm_matmul_workspace_size(R.RMM_BF16, M, D, F, 0.8), dtype=torch.uint8, device=dev)
    dws = torch.empty(R.rmm_matmul_workspace_size(R.RMM_BF16, M, F, D, 0.5), dtype=torch.uint8, device=dev)

    def block(ev):
        ev[0].record(stream)
        R.rmm_mlp_block(X, Wu, Wg, Wd, 0.8, 0.5, out=Y, ws=bws)
        ev[1].record(stream)

    def chain(ev):
        ev[0].record(stream)
        R.rmm_matmul(X, Wu, 0.8, out=U, ws=uws)
        R.rmm_matmul(X, Wg, 0.8, out=G, ws=uws)
        H = torch.nn.functional.silu(G) * U
        R.rmm_matmul(H, Wd, 0.5, out=Y, ws=dws)
        ev[1].record(stream)

    def dense(ev):
        ev[0].record(stream)
        torch.matmul(torch.nn.functional.silu(X @ Wg) * (X @ Wu), Wd, out=Y)
        ev[1].record(stream)
    for _ in range(3):
        for f in (block, chain, dense):
            f([torch.cuda.Event(enable_timing=True) for _ in range(2)])
    bl = statistics.mean(p[0] for p in timed(block, steps, 2))
    ch = statistics.mean(p[0] for p in timed(chain, steps, 2))
    de = statistics.mean(p[0] for p in timed(dense, steps, 2))
    red_flops = 2.0 * M * F * R.rmm_k_from_rho(0.8, D) * 2 + 2.0 * M * D * R.rmm_k_from_rho(0.5, F)
    out["mlp_block"] = {"block_us": bl * 1e3, "chain_of_rmm_matmul_us": ch * 1e3, "dense_cublas_us": de * 1e3,
                        "speedup_vs_dense": de / bl, "effective_tflops": red_flops / (bl * 1e-3) / 1e12,
                        "gpu_launches_per_call": 11}
    if R.rmm_device_error(stream) != 0:
        raise SystemExit("device error during the block runs")
    out["workload"] = (f"X[{M}x{D}] bf16 (MLP up/gate activation); q/k/v-shaped W at rho 0.5; gated MLP "
                       f"d_ff={F}, rho_up=0.8, rho_down=0.5; 256 MiB flush between steps")
    return out


def rho_sweep(R, A, B, rhos, dense_ms, steps, timed, stream, dev):
    """The same step (rmm_matmul, same flush protocol) at other rho values of
    one workload, next to its dense product.  A failure is reported in the
    entry of its rho, so it cannot cost the rest of the line."""
    import torch
    M, d = A.shape
    N = B.shape[1]
    out = {}
    try:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    except Exception as e:  # noqa: BLE001 - reported in the line
        return {"error": f"{type(e).__name__}: {e}"[:200]}
    for rho in rhos:
        try:
            k = R.rmm_k_from_rho(rho, d)
            ws = torch.empty(R.rmm_matmul_workspace_size(R.RMM_BF16, M, d, N, rho), dtype=torch.uint8, device=dev)

            def step(ev, rho=rho, ws=ws):
                ev[0].record(stream)
                R.rmm_matmul(A, B, rho, out=Y, ws=ws)
                ev[1].record(stream)
            for _ in range(3):
                step([torch.cuda.Event(enable_timing=True) for _ in range(2)])
            ms = statistics.mean(p[0] for p in timed(step, steps, 2))
            if R.rmm_device_error(stream) != 0:
                raise RuntimeError("device error word set")
            out[f"rho={rho}"] = {"k": k, "step_us": ms * 1e3, "effective_tflops": 2.0 * M * N * k / (ms * 1e-3) / 1e12,
                                 "speedup_vs_dense": dense_ms / ms}
        except Exception as e:  # noqa: BLE001 - reported in the line
            out[f"rho={rho}"] = {"error": f"{type(e).__name__}: {e}"[:200]}
    return out


def measure_down(R, workloads, bf16_tensor, dev, stream, flush, steps, timed):
    """The MLP down projection H [4096 x 14336] . W [14336 x 4096] at rho = 0.5
    (H = SiLU(G) * U formed in fp64 and rounded): the config where the
    selection reads the widest activation.  The same step and protocol as the
    headline (rmm_matmul, 256 MiB flush between steps), next to cuBLAS."""
    import torch
    inp = workloads.mlp_down()
    Hd, Wd = bf16_tensor(inp.A, dev), bf16_tensor(inp.B, dev)
    Md, dd, Nd = inp.M, inp.d, inp.N
    k = R.rmm_k_from_rho(0.5, dd)
    Y = torch.empty((Md, Nd), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(R.rmm_matmul_workspace_size(R.RMM_BF16, Md, dd, Nd, 0.5), dtype=torch.uint8, device=dev)
    ss = torch.empty(dd, dtype=torch.float32, device=dev)
    idx = torch.empty(k, dtype=torch.int32, device=dev)
    sws = torch.empty(max(R.rmm_score_workspace_size(R.RMM_BF16, 1, Md, dd), 256), dtype=torch.uint8, device=dev)

    def rmm(ev):
        ev[0].record(stream)
        R.rmm_matmul(Hd, Wd, 0.5, out=Y, ws=ws)
        ev[1].record(stream)

    def select(ev):
        ev[0].record(stream)
        R.rmm_score(Hd, out=ss, ws=sws)
        R.rmm_topk(ss, k, out=idx)
        ev[1].record(stream)

    def dense(ev):
        ev[0].record(stream)
        torch.matmul(Hd, Wd, out=Y)
        ev[1].record(stream)
    for _ in range(3):
        rmm([torch.cuda.Event(enable_timing=True) for _ in range(2)])
        dense([torch.cuda.Event(enable_timing=True) for _ in range(2)])
        select([torch.cuda.Event(enable_timing=True) for _ in range(2)])
    ms = statistics.mean(p[0] for p in timed(rmm, steps, 2))
    dms = statistics.mean(p[0] for p in timed(dense, steps, 2))
    sel_ms = statistics.mean(p[0] for p in timed(select, steps, 2))
    if R.rmm_device_error(stream) != 0:
        raise SystemExit("device error during the down-projection runs")
    sweep = rho_sweep(R, Hd, Wd, (0.8, 1.0), dms, min(steps, 30), timed, stream, dev)
    return {"workload": f"MLP down projection H[{Md}x{dd}] . W[{dd}x{Nd}] bf16, rho=0.5, 256 MiB flush between steps",
            "step_us": ms * 1e3, "dense_us": dms * 1e3, "speedup_vs_dense": dms / ms,
            "effective_tflops": 2.0 * Md * Nd * k / (ms * 1e-3) / 1e12, "other_rho": sweep,
            "select_overhead": {"score_topk_us": sel_ms * 1e3, "dense_us": dms * 1e3, "frac_of_dense": sel_ms / dms,
                                "target": 0.10}}


DEC_ATTN = {"seed": 5, "Hq": 32, "Hkv": 8, "L": 32768, "D": 128, "rho_d": 0.5, "rho_t": 0.5}


def measure_decode_attention(R, workloads, bf16_tensor, dev, stream, steps, timed, hbm_gbs):
    """One decode step of reduced attention (GQA 32/8 heads, D = 128, a 32768-token
    cache) for 1 and 8 sequences, next to torch's SDPA on the full cache.
    Bandwidth counts the algorithmic bytes: every key row (the head_dim
    selection differs per q-head, so every key sector is needed), the union
    over a kv-group's q-heads of their kept value rows, q and O."""
    import numpy as np
    import torch
    a = DEC_ATTN
    out = {}
    for B in (1, 8):
        inp = workloads.decode_attention(a["seed"], B, a["Hq"], a["Hkv"], a["L"], a["D"], a["rho_d"], a["rho_t"])
        q, K, V = (bf16_tensor(x, dev) for x in (inp.q, inp.K, inp.V))
        kt = R.rmm_k_from_rho(a["rho_t"], a["L"])
        O = torch.empty((B, a["Hq"], a["D"]), dtype=torch.bfloat16, device=dev)
        idx_t = torch.empty((B * a["Hq"], kt), dtype=torch.int32, device=dev)
        ws = torch.empty(R.rmm_decode_attention_workspace_size(B, a["Hq"], a["L"], a["D"], a["rho_t"], False, False),
                         dtype=torch.uint8, device=dev)

        def rmm(ev):
            ev[0].record(stream)
            R.rmm_decode_attention(q, K, V, a["L"], a["rho_d"], a["rho_t"], out=O, ws=ws)
            ev[1].record(stream)
        q4 = q.view(B, a["Hq"], 1, a["D"])

        def sdpa(ev):
            ev[0].record(stream)
            torch.nn.functional.scaled_dot_product_attention(q4, K, V, enable_gqa=True)
            ev[1].record(stream)
        for _ in range(3):
            rmm([torch.cuda.Event(enable_timing=True) for _ in range(2)])
            sdpa([torch.cuda.Event(enable_timing=True) for _ in range(2)])
        rmm_us = statistics.mean(p[0] for p in timed(rmm, steps, 2)) * 1e3
        sdpa_us = statistics.mean(p[0] for p in timed(sdpa, steps, 2)) * 1e3
        # the kept lists (an optional output, not asked for in the timed calls)
        R.rmm_decode_attention(q, K, V, a["L"], a["rho_d"], a["rho_t"], out=O, idx_t=idx_t, ws=ws)
        it = idx_t.cpu().numpy().reshape(B, a["Hkv"], a["Hq"] // a["Hkv"], kt)
        union = sum(len(np.unique(it[b, g])) for b in range(B) for g in range(a["Hkv"]))
        row = a["D"] * 2
        alg = B * a["Hkv"] * a["L"] * row + union * row + 2 * B * a["Hq"] * row
        gbs = alg / (rmm_us * 1e-6) / 1e9
        out[f"B{B}"] = {"rmm_us": rmm_us, "sdpa_us": sdpa_us, "speedup_vs_sdpa": sdpa_us / rmm_us,
                        "algorithmic_MB": alg / 1e6, "GB/s": gbs, "frac_hbm": gbs / hbm_gbs,
                        "kept_value_rows_union_frac": union / (B * a["Hkv"] * a["L"]), "gpu_launches_per_call": 3}
    if R.rmm_device_error(stream) != 0:
        raise SystemExit("device error during the decode-attention runs")
    out["workload"] = (f"decode step: q[B x {a['Hq']} x {a['D']}] over K/V caches [B x {a['Hkv']} x {a['L']} x "
                       f"{a['D']}] bf16, rho_d={a['rho_d']} rho_t={a['rho_t']}; caches larger than L2 (B=8), "
                       "256 MiB write flush between steps")
    return out


def run_rmm(args):
    import numpy as np
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    import input_adaptive_reduced_score_b200 as R
    import workloads
    from tests.helpers import bf16_tensor

    dev = torch.device("cuda", local_rank)
    k = R.rmm_k_from_rho(RHO, D)
    X = bf16_tensor(workloads.llm_activation_bf16(1 + 101 * rank, M, D), dev)
    Wt = bf16_tensor(workloads.weight_bf16(1, D, N), dev)
    ss = torch.empty(D, dtype=torch.float32, device=dev)
    idx = torch.empty(k, dtype=torch.int32, device=dev)
    AI = torch.empty((M, (k + 7) // 8 * 8), dtype=torch.bfloat16, device=dev)[:, :k]
    BI = torch.empty((k, N), dtype=torch.bfloat16, device=dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    sws_n = R.rmm_score_workspace_size(R.RMM_BF16, 1, M, D)
    sws = torch.empty(max(sws_n, 256), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    gws = torch.empty(R.rmm_gemm_workspace_size(R.RMM_BF16, N, k), dtype=torch.uint8, device=dev)
    # rmm_matmul: score (one cluster launch for aligned bf16), top-k, one
    # launch compacting A and copying the first column blocks of the kept
    # rows of B (zeroing the copy counters), the tensor-core product whose
    # spare warps copy the rest of B's kept rows while it multiplies
    launches_per_step = 4
    kernel_calls = {
        "score": lambda: R.rmm_score(X, out=ss, ws=sws),
        "topk": lambda: R.rmm_topk(ss, k, out=idx),
        "compact": lambda: R.rmm_compact(X, idx, out=AI),
        "gemm": lambda: R.rmm_gemm(AI, Wt, idx, out=Y, ws=gws),
    }
    # the timed step: the whole path as one call
    mws_step = torch.empty(R.rmm_matmul_workspace_size(R.RMM_BF16, M, D, N, RHO), dtype=torch.uint8, device=dev)
    whole_path_call = lambda: R.rmm_matmul(X, Wt, RHO, out=Y, idx_out=idx, ws=mws_step)
    # the earlier form: both operands in one launch, then the product on them
    two_launch_calls = [
        kernel_calls["score"], kernel_calls["topk"],
        lambda: R.rmm_compact_gather(X, Wt, idx, out_a=AI, out_b=BI),
        lambda: R.rmm_gemm_compacted(AI, BI, out=Y),
    ]

    def step(ev=None):
        # Kernels are launched with programmatic dependent launch: each one's
        # launch and set-up overlap its predecessor's tail.  An event recorded
        # between two kernels ends that overlap, so the timed step records only
        # the events the GEMM's own duration needs.
        if ev is not None:
            ev[0].record(stream)
        kernel_calls["score"]()
        kernel_calls["topk"]()
        kernel_calls["compact"]()
        if ev is not None:
            ev[1].record(stream)
        kernel_calls["gemm"]()
        if ev is not None:
            ev[2].record(stream)

    def step_serialised(ev):
        # per-kernel breakdown (an event between every pair of kernels)
        ev[0].record(stream)
        for j, fn in enumerate(kernel_calls.values()):
            fn()
            ev[j + 1].record(stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    def timed(fn, steps, nev):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(steps)]
        barrier()
        torch.cuda.synchronize(dev)
        for i in range(steps):
            flush.zero_()
            fn(evs[i])
        torch.cuda.synchronize(dev)
        barrier()
        return [[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(nev - 1)] for i in range(steps)]

    def whole_path_step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        whole_path_call()
        if ev is not None:
            ev[1].record(stream)

    def two_launch_step(ev):
        ev[0].record(stream)
        for fn in two_launch_calls:
            fn()
        ev[1].record(stream)

    def select_step(ev):
        # the selection alone: column scores and top-k, one event interval
        ev[0].record(stream)
        kernel_calls["score"]()
        kernel_calls["topk"]()
        ev[1].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        whole_path_step()
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    if R.rmm_device_error(stream) != 0:
        raise SystemExit("device error during warm-up")

    # The timed steps are rmm_matmul calls (no event inside a step, so every
    # kernel's launch overlaps its predecessor).  The GEMM's own duration for
    # the roofline comes from the same path split into its public calls with
    # an event before rmm_gemm, timed right after under the same clock record.
    remeasured = False
    for attempt in range(2):
        with ClockSampler(torch.cuda.get_device_properties(dev)) as clk:
            per = timed(whole_path_step, args.steps, 2)
            split = timed(step, min(args.steps, 100), 3)
        if not clk.rejected():
            break
        remeasured = True
    if R.rmm_device_error(stream) != 0:
        raise SystemExit("device error during the timed steps")
    step_ms = [p[0] for p in per]
    stage_ms = {"select_and_compact": statistics.mean(p[0] for p in split),
                "gemm": statistics.mean(p[1] for p in split)}
    split_ms = statistics.mean(sum(p) for p in split)
    ser = timed(step_serialised, min(args.steps, 50), len(kernel_calls) + 1)
    serial_ms = {name: statistics.mean(p[j] for p in ser) for j, name in enumerate(kernel_calls)}
    for _ in range(3):
        two_launch_step([torch.cuda.Event(enable_timing=True) for _ in range(2)])
    two_launch_ms = statistics.mean(p[0] for p in timed(two_launch_step, min(args.steps, 50), 2))
    local_ms = sum(step_ms)
    flops_step = 2.0 * M * N * k
    tot_ms, tot_flops = aggregate(local_ms, flops_step * args.steps, world)
    value = tot_flops / (tot_ms * 1e-3) / 1e12

    # dense cuBLAS bf16 at the same shape, same flush protocol
    def dense(ev):
        ev[0].record(stream)
        torch.matmul(X, Wt, out=Y)
        ev[1].record(stream)
    for _ in range(3):
        torch.matmul(X, Wt, out=Y)
    dense_ms = statistics.mean(p[0] for p in timed(dense, min(args.steps, 100), 2))
    for _ in range(3):
        select_step([torch.cuda.Event(enable_timing=True) for _ in range(2)])
    select_ms = statistics.mean(p[0] for p in timed(select_step, min(args.steps, 100), 2))
    # the same workload at the other rho values of the up-projection config
    other_rho = rho_sweep(R, X, Wt, (0.7, 0.8, 1.0), dense_ms, min(args.steps, 30), timed, stream, dev)

    # end to end through the public API, every step moving its X in from
    # pinned host memory and its Y out to pinned host memory.  Steps are
    # pipelined over three streams with two device buffers each: step i's X
    # is copied in while step i-1 computes and step i-2's Y is copied out
    # (the copies use the two PCIe directions and the copy engines; each step
    # still writes the 256 MiB flush before its product).  Time = events
    # around the whole sequence / steps.
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    Xh = [X.cpu().pin_memory() for _ in range(2)]
    Yh = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    Xd = [torch.empty_like(X) for _ in range(2)]
    Yd = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    mws = torch.empty(R.rmm_matmul_workspace_size(R.RMM_BF16, M, D, N, RHO), dtype=torch.uint8, device=dev)

    def e2e_pipeline(K):
        ev = [[torch.cuda.Event() for _ in range(3)] for _ in range(K)]  # in, compute, out
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        t0.record(stream)
        for i in range(K):
            b = i % 2
            s_in.wait_event(t0 if i < 2 else ev[i - 2][1])  # compute i-2 has read Xd[b]
            with torch.cuda.stream(s_in):
                Xd[b].copy_(Xh[b], non_blocking=True)
            ev[i][0].record(s_in)
            stream.wait_event(ev[i][0])
            if i >= 2:
                stream.wait_event(ev[i - 2][2])  # copy-out i-2 has read Yd[b]
            flush.zero_()
            R.rmm_matmul(Xd[b], Wt, RHO, out=Yd[b], ws=mws, stream=stream)
            ev[i][1].record(stream)
            s_out.wait_event(ev[i][1])
            with torch.cuda.stream(s_out):
                Yh[b].copy_(Yd[b], non_blocking=True)
            ev[i][2].record(s_out)
        stream.wait_event(ev[K - 1][2])
        t1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        return t0.elapsed_time(t1)
    e2e_pipeline(3)
    e2e_total_ms = e2e_pipeline(args.e2e_steps)
    e2e_tot, e2e_flops = aggregate(e2e_total_ms, flops_step * args.e2e_steps, world)
    e2e_value = e2e_flops / (e2e_tot * 1e-3) / 1e12
    if R.rmm_device_error(stream) != 0:
        raise SystemExit("device error during the dense / end-to-end runs")

    peaks, peak_src = load_peaks()
    attention = measure_attention(R, workloads, bf16_tensor, dev, stream, flush, min(args.steps, 20), timed, peaks)
    attention_gqa = measure_attention(R, workloads, bf16_tensor, dev, stream, flush, min(args.steps, 10), timed,
                                      peaks, ATTN_GQA)
    layer70b = measure_layer70b(R, workloads, bf16_tensor, dev, stream, flush, min(args.steps, 20), timed, peaks)
    decode = measure_decode(R, workloads, bf16_tensor, dev, stream, flush, min(args.steps, 50), timed, Wt,
                            peaks["hbm_gbs"])
    w8 = measure_w8(R, workloads, bf16_tensor, dev, stream, flush, min(args.steps, 50), timed, X, peaks["hbm_gbs"])
    dec_attn = measure_decode_attention(R, workloads, bf16_tensor, dev, stream, min(args.steps, 30), timed,
                                        peaks["hbm_gbs"])
    block = measure_block(R, workloads, bf16_tensor, dev, stream, flush, min(args.steps, 30), timed, X)
    down = measure_down(R, workloads, bf16_tensor, dev, stream, flush, min(args.steps, 50), timed)
    gemm_ms = stage_ms["gemm"]
    achieved = flops_step / (gemm_ms * 1e-3) / 1e12
    # the GEMM is timed inside a loop of seconds: when the power cap acted
    # during it, the sustained (power-capped) cuBLAS figure is its peak
    capped = "sw_power_cap" in clk.summary()["reasons"]
    peak = peaks["bf16_tflops_sustained"] if capped else peaks["bf16_tflops"]
    peak_label = (f"{peak_src} sustained bf16 (sw_power_cap active during the timed steps)" if capped
                  else f"{peak_src} burst bf16 (no power cap during the timed steps)")
    traffic = traffic_per_launch()
    hbm = peaks["hbm_gbs"]
    # algorithmic bytes per launch: score reads A; top-k reads the d scores and
    # writes k indices; compaction reads A (at half density every 32-byte
    # sector holds a kept column) and writes A_I
    kbytes = {"score": 2.0 * M * D, "topk": 4.0 * D + 4.0 * k, "compact": 2.0 * M * D + 2.0 * M * k}
    kernels = {"split_step_us": {name: v * 1e3 for name, v in stage_ms.items()},
               "split_step_total_us": split_ms * 1e3,
               "two_launch_gather_step_us": two_launch_ms * 1e3}
    for name, v in serial_ms.items():
        us = v * 1e3
        if name == "gemm":
            kernels[name] = {"us_serialised": us, "TFLOP/s": flops_step / (v * 1e-3) / 1e12}
        else:
            gbs = kbytes[name] / (v * 1e-3) / 1e9
            kernels[name] = {"us_serialised": us, "GB/s": gbs, "frac_hbm": gbs / hbm}
    path_ms = statistics.mean(step_ms)
    min_bytes = 2.0 * M * D + 2.0 * k * N + 2.0 * M * N
    path_roof_ms = max(flops_step / (peaks["bf16_tflops"] * 1e12), min_bytes / (hbm * 1e9)) * 1e3

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": tot_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded Philox inputs of the workload's shape and distribution)",
            "config": bench_config(world),
            "speedup_vs_dense": dense_ms / path_ms, "dense_ms": dense_ms, "other_rho": other_rho,
            "select_overhead_frac_of_dense": select_ms / dense_ms,
            "select_overhead": {"score_topk_us": select_ms * 1e3, "dense_us": dense_ms * 1e3,
                                "frac_of_dense": select_ms / dense_ms, "target": 0.10,
                                "mlp_down": down["select_overhead"]},
            "dense_tflops": 2.0 * M * N * D / (dense_ms * 1e-3) / 1e12,
            "dense_equivalent_tflops": 2.0 * M * N * D / (path_ms * 1e-3) / 1e12,
            "path_roofline_frac": path_roof_ms / path_ms,
            "roofline": {"kernel": "rmm_gemm: first-wave row copy + gemm_bf16_tc_pair_kernel<true> (copies the rest)",
                         "bound": "tensor", "achieved": achieved,
                         "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                         "peak_source": peak_label, "frac_of_burst": achieved / peaks["bf16_tflops"],
                         "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"]},
            "kernels": kernels,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": int(X.numel() * 2),
                    "d2h_bytes_per_step": int(Y.numel() * 2), "api": "rmm_matmul",
                    "ms_per_step": e2e_tot / args.e2e_steps,
                    "schedule": "steps pipelined over copy-in, compute and copy-out streams (double buffers)"},
            "gpu_launches": launches_per_step * args.steps,
            "attention": attention,
            "attention_gqa32k": attention_gqa,
            "layer70b": layer70b,
            "decode": decode,
            "int8_weight": w8,
            "decode_attention": dec_attn,
            "block_driver": block,
            "mlp_down": down,
            "clocks": clk.summary(), "clock_remeasured": remeasured,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = time_cpu_oracle()
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def run_case(case):
    """Short runs for profiler captures: the timed matmul step four times, the
    reduced-attention workload three times, the decode products (1 and 16
    rows on the MLP up/gate weight) twelve times each with a 256 MiB write in
    between, and so on for the other workloads."""
    import numpy as np
    import torch
    import input_adaptive_reduced_score_b200 as R
    import workloads
    from tests.helpers import bf16_tensor
    dev = torch.device("cuda", 0)
    if case == "matmul":
        # the timed step: rmm_matmul on the MLP up/gate workload, four calls
        # with a 256 MiB write before each
        X = bf16_tensor(workloads.llm_activation_bf16(1, M, D), dev)
        Wt = bf16_tensor(workloads.weight_bf16(1, D, N), dev)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(R.rmm_matmul_workspace_size(R.RMM_BF16, M, D, N, RHO), dtype=torch.uint8, device=dev)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        for _ in range(4):
            flush.zero_()
            R.rmm_matmul(X, Wt, RHO, out=Y, ws=ws)
    elif case == "layer70b":
        # every projection of the 70B-shaped layer, rmm_matmul twice each
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        for name, Mg, dg, Ng, rho in workloads.layer70b_gemms():
            inp = workloads.layer70b_inputs(name)
            X, Wt = bf16_tensor(inp.A, dev), bf16_tensor(inp.B, dev)
            Y = torch.empty((Mg, Ng), dtype=torch.bfloat16, device=dev)
            for _ in range(2):
                flush.zero_()
                R.rmm_matmul(X, Wt, rho, out=Y)
            del X, Wt, Y
    elif case == "down":
        inp = workloads.mlp_down()
        Hd, Wd = bf16_tensor(inp.A, dev), bf16_tensor(inp.B, dev)
        Y = torch.empty((inp.M, inp.N), dtype=torch.bfloat16, device=dev)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        for _ in range(4):
            flush.zero_()
            R.rmm_matmul(Hd, Wd, 0.5, out=Y)
    elif case in ("attention", "attention_gqa"):
        a = ATTN if case == "attention" else ATTN_GQA
        inp = workloads.attention(a["seed"], a["B"], a["Hq"], a["Hkv"], a["S"], a["D"], a["rho_d"], a["rho_t"])
        Q, K, V = (bf16_tensor(x, dev) for x in (inp.Q, inp.K, inp.V))
        O = torch.empty_like(Q)
        ws = torch.empty(R.rmm_attention_workspace_size(a["B"], a["Hq"], a["Hkv"], a["S"], a["D"], a["rho_d"],
                                                        a["rho_t"]), dtype=torch.uint8, device=dev)
        for _ in range(3):
            R.rmm_attention(Q, K, V, a["rho_d"], a["rho_t"], out=O, ws=ws)
    elif case == "block":
        X = bf16_tensor(workloads.llm_activation_bf16(1, M, D), dev)
        Ws = [bf16_tensor(workloads.weight_bf16(9, D, n, group=i), dev) for i, n in enumerate((D, 1024, 1024))]
        F = 14336
        Wu = bf16_tensor(workloads.weight_bf16(10, D, F, group=0), dev)
        Wg = bf16_tensor(workloads.weight_bf16(10, D, F, group=1), dev)
        Wd = bf16_tensor(workloads.weight_bf16(10, F, D, group=2), dev)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        for _ in range(3):
            flush.zero_()
            R.rmm_matmul_multi(X, Ws, 0.5)
            flush.zero_()
            R.rmm_mlp_block(X, Wu, Wg, Wd, 0.8, 0.5)
    elif case == "topk":
        # the top-k on its own, at the row counts and lengths the paths give
        # it: one row of 4096 and of 14336 scores (the MLP up and down
        # projections), 32 rows of 32768 (a decode step's token top-k, one
        # sequence) and 256 such rows (eight sequences); k = d / 2
        gen = torch.Generator(device=dev).manual_seed(3)
        for rows, d in ((1, 4096), (1, 14336), (32, 32768), (256, 32768)):
            sc = torch.randn(rows, d, device=dev, generator=gen)
            out = torch.empty(rows, d // 2, dtype=torch.int32, device=dev)
            for _ in range(3):
                R.rmm_topk(sc, d // 2, out=out)
    elif case == "decode_attention":
        a = DEC_ATTN
        for B in (1, 8):
            inp = workloads.decode_attention(a["seed"], B, a["Hq"], a["Hkv"], a["L"], a["D"], a["rho_d"], a["rho_t"])
            q, K, V = (bf16_tensor(x, dev) for x in (inp.q, inp.K, inp.V))
            O = torch.empty((B, a["Hq"], a["D"]), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(R.rmm_decode_attention_workspace_size(B, a["Hq"], a["L"], a["D"], a["rho_t"]),
                             dtype=torch.uint8, device=dev)
            for _ in range(3):
                R.rmm_decode_attention(q, K, V, a["L"], a["rho_d"], a["rho_t"], out=O, ws=ws)
    elif case == "w8":
        q, sc = workloads.weight_int8(1, D, N)
        Wq, S = torch.from_numpy(q).to(dev), torch.from_numpy(sc).to(dev)
        X = bf16_tensor(workloads.llm_activation_bf16(1, M, D), dev)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        for _ in range(3):
            flush.zero_()
            R.rmm_matmul_w8(X, Wq, S, RHO, out=Y)
        k = R.rmm_k_from_rho(RHO, D)
        idx = torch.from_numpy(np.sort(np.random.default_rng(0).choice(D, k, replace=False)).astype(np.int32)).to(dev)
        for rows in (1, 16):
            AI = R.rmm_compact(bf16_tensor(workloads.llm_activation_bf16(7, rows, D), dev), idx)
            Yr = torch.empty((rows, N), dtype=torch.bfloat16, device=dev)
            for _ in range(12):
                flush.zero_()
                R.rmm_gemm_w8(AI, Wq, S, idx, out=Yr)
    else:
        k = R.rmm_k_from_rho(RHO, D)
        Wt = bf16_tensor(workloads.weight_bf16(1, D, N), dev)
        idx = torch.from_numpy(np.sort(np.random.default_rng(0).choice(D, k, replace=False)).astype(np.int32)).to(dev)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        gws = torch.empty(R.rmm_gemm_workspace_size(R.RMM_BF16, N, k), dtype=torch.uint8, device=dev)
        for rows in (1, 16):
            AI = R.rmm_compact(bf16_tensor(workloads.llm_activation_bf16(7, rows, D), dev), idx)
            Y = torch.empty((rows, N), dtype=torch.bfloat16, device=dev)
            for _ in range(12):
                flush.zero_()
                R.rmm_gemm(AI, Wt, idx, out=Y, ws=gws)
    torch.cuda.synchronize()
    if R.rmm_device_error() != 0:
        raise SystemExit("device error")


def main():
    args = parse_args()
    if args.case != "bench":
        run_case(args.case)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus and not (args.impl == "reference"):
        if world == 1 and args.gpus > 1:
            raise SystemExit("for --gpus > 1 launch with torch.distributed.run (one rank per GPU)")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_rmm(args)


if __name__ == "__main__":
    main()
