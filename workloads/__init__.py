"""Seeded synthetic inputs for the reduced-matmul and reduced-attention workloads.

This module draws random numbers and stores them in the exact element formats
that both the CPU oracle and the CUDA path read.  It holds none of the
method's arithmetic: no column norms, no selection, no products.  Both sides
consume the buffers it returns; neither side shares any other code.

Generator: numpy's Philox-4x32-10 counter-based bit generator, one independent
substream per (seed, tensor id, head group, attempt), keyed as documented in
``substream``.  Normals are numpy's standard normals drawn in fp64.

bf16 storage: values are rounded fp64 -> fp32 -> bf16 with round-to-nearest-even
and kept as raw uint16 bit patterns (numpy has no bf16 dtype).

Workload shapes and distributions follow the five synthetic configurations of
the benchmark (names below are by what they are, with their sizes).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# ---------------------------------------------------------------- bf16 codec


def f32_to_bf16_bits(x) -> np.ndarray:
    """Round finite fp32 (or wider) values to bf16, nearest-even; return uint16 bits."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    if not np.isfinite(f).all():
        raise ValueError("bf16 encoding: non-finite input")
    # (u + 0x7FFF + lsb) >> 16 on the fp32 bit pattern u, where lsb is bit 16
    # (ties to even).  Finite patterns are at most 0xFF7FFFFF, so the sum
    # stays below 2^32 and uint32 arithmetic is exact.
    u = f.view(np.uint32)
    r = u >> 16
    r &= 1
    r += 0x7FFF
    r += u
    r >>= 16
    return r.astype(np.uint16)


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact decode of bf16 bit patterns to fp64."""
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_bits_to_f32(bits) -> np.ndarray:
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- substreams

TENSOR_IDS = {
    "A": 1, "B": 2, "X": 3, "W": 4, "G": 5, "U": 6, "Q": 7, "K": 8, "V": 9,
    "colscale": 10, "outliers": 11, "qscale": 12, "kscale": 13, "vscale": 14, "W8": 15,
}


def substream(seed: int, tensor: str, group: int = 0, attempt: int = 0) -> np.random.Generator:
    """Independent Philox stream for one tensor.

    Key (128 bits) = seed << 64 | tensor_id << 48 | group << 16 | attempt.
    """
    tid = TENSOR_IDS[tensor]
    if not (0 <= group < (1 << 32) and 0 <= attempt < (1 << 16)):
        raise ValueError("substream: group/attempt out of range")
    key = (int(seed) << 64) | (tid << 48) | (int(group) << 16) | int(attempt)
    return np.random.Generator(np.random.Philox(key=key))


# ---------------------------------------------------------------- workloads


@dataclass
class MatmulInputs:
    """A [M x d] activation and B [d x N] weight, row-major.

    ``dtype`` is "f32" (arrays are np.float32) or "bf16" (arrays are uint16 bits).
    ``rhos`` are the retention ratios the workload is quoted at.
    """
    name: str
    dtype: str
    A: np.ndarray
    B: np.ndarray
    rhos: tuple
    seed: int
    meta: dict = field(default_factory=dict)

    @property
    def M(self):
        return self.A.shape[0]

    @property
    def d(self):
        return self.A.shape[1]

    @property
    def N(self):
        return self.B.shape[1]


def _normal(g: np.random.Generator, shape) -> np.ndarray:
    return g.standard_normal(size=shape, dtype=np.float64)


def tiny_fp32(seed: int = 0, M: int = 64, d: int = 256, N: int = 128) -> MatmulInputs:
    """Single reduced matmul, fp32: A = Z * diag(10^U(-1,1)) (log-uniform column
    scale in [0.1, 10]), B ~ N(0, 1/d)."""
    gs = substream(seed, "colscale")
    scale = 10.0 ** gs.uniform(-1.0, 1.0, size=d)
    A = (_normal(substream(seed, "A"), (M, d)) * scale[None, :]).astype(np.float32)
    B = (_normal(substream(seed, "B"), (d, N)) * (1.0 / math.sqrt(d))).astype(np.float32)
    return MatmulInputs(f"reduced matmul fp32 {M}x{d}x{N}", "f32", A, B, (0.5,), seed)


def llm_activation_bf16(seed: int, tokens: int, hidden: int, outlier_frac: float = 0.01,
                        outlier_gain: float = 20.0, group: int = 0) -> np.ndarray:
    """Activation X [tokens x hidden]: N(0,1) times a per-channel lognormal(0,1)
    scale, with round(outlier_frac*hidden) channels (uniform, without
    replacement) multiplied by outlier_gain.  Returns bf16 bits."""
    scale = np.exp(_normal(substream(seed, "colscale", group), hidden))
    n_out = int(round(outlier_frac * hidden))
    if n_out:
        ch = substream(seed, "outliers", group).choice(hidden, size=n_out, replace=False)
        scale[ch] *= outlier_gain
    X = _normal(substream(seed, "X", group), (tokens, hidden)) * scale[None, :]
    return f32_to_bf16_bits(X)


def weight_bf16(seed: int, rows: int, cols: int, std: float = 0.02, group: int = 0) -> np.ndarray:
    """Weight [rows x cols] ~ N(0, std^2), bf16 bits, row-major (rows = contraction dim)."""
    return f32_to_bf16_bits(_normal(substream(seed, "W", group), (rows, cols)) * std)


def mlp_up(seed: int = 1, tokens: int = 4096, hidden: int = 4096, ffn: int = 14336) -> MatmulInputs:
    """MLP up/gate projection, bf16: X [tokens x hidden] (per-channel lognormal
    scale, 1% outlier channels x20) times W [hidden x ffn] ~ N(0, 0.02^2)."""
    X = llm_activation_bf16(seed, tokens, hidden)
    W = weight_bf16(seed, hidden, ffn)
    return MatmulInputs(f"MLP up/gate projection {tokens}x{hidden}x{ffn} bf16", "bf16", X, W,
                        (0.5, 0.7, 0.8, 1.0), seed)


def silu(x):
    return x / (1.0 + np.exp(-x))


def mlp_down(seed: int = 2, tokens: int = 4096, ffn: int = 14336, hidden: int = 4096) -> MatmulInputs:
    """MLP down projection, bf16: H = SiLU(G) * U with G, U ~ N(0,1) formed in
    fp64 then rounded, times W [ffn x hidden] ~ N(0, 0.02^2)."""
    G = _normal(substream(seed, "G"), (tokens, ffn))
    U = _normal(substream(seed, "U"), (tokens, ffn))
    H = f32_to_bf16_bits(silu(G) * U)
    del G, U
    W = weight_bf16(seed, ffn, hidden)
    return MatmulInputs(f"MLP down projection {tokens}x{ffn}x{hidden} bf16", "bf16", H, W,
                        (0.5, 0.8, 1.0), seed)


def layer70b_gemms(seed: int = 4, tokens: int = 2048, hidden: int = 8192, mlp: int = 28672,
                   n_q_heads: int = 64, n_kv_heads: int = 8, head_dim: int = 128):
    """Shapes of the 70B-class layer: (name, M, d, N, rho) per projection.

    Each projection's activation is drawn independently (a shape benchmark,
    not a chained layer); use ``layer70b_inputs`` to materialise one."""
    kv = n_kv_heads * head_dim
    return [
        ("q_proj", tokens, hidden, hidden, 0.5),
        ("k_proj", tokens, hidden, kv, 0.5),
        ("v_proj", tokens, hidden, kv, 0.5),
        ("o_proj", tokens, hidden, hidden, 0.5),
        ("up_proj", tokens, hidden, mlp, 0.8),
        ("gate_proj", tokens, hidden, mlp, 0.8),
        ("down_proj", tokens, mlp, hidden, 0.8),
    ]


def layer70b_inputs(which: str, seed: int = 4, **kw) -> MatmulInputs:
    shapes = {n: (M, d, N, r) for n, M, d, N, r in layer70b_gemms(seed, **kw)}
    M, d, N, rho = shapes[which]
    group = list(shapes).index(which) + 1
    X = llm_activation_bf16(seed, M, d, group=group)
    W = weight_bf16(seed, d, N, group=group)
    return MatmulInputs(f"70B layer {which} {M}x{d}x{N} bf16", "bf16", X, W, (rho,), seed)


def scaled_matmul_bf16(seed: int, M: int, d: int, N: int, rhos=(0.5,), outlier_frac=0.01) -> MatmulInputs:
    """Generic bf16 case with the up-projection distribution at any shape
    (used for ragged-shape parity cases)."""
    X = llm_activation_bf16(seed, M, d, outlier_frac=outlier_frac)
    W = weight_bf16(seed, d, N, std=0.02)
    return MatmulInputs(f"bf16 {M}x{d}x{N}", "bf16", X, W, tuple(rhos), seed)


def weight_int8(seed: int, rows: int, cols: int, std: float = 0.02, group: int = 0):
    """Int8 weight [rows x cols] with one fp32 scale per column, stored the way
    a symmetric absmax quantiser stores an N(0, std^2) weight:
    scale[n] = max_j |W[j, n]| / 127 (rounded to fp32), q = W / scale[n]
    rounded half-to-even and clipped to [-127, 127].  Returns (q int8, scale
    fp32).  Weight storage format only; nothing of the reduced product."""
    W = _normal(substream(seed, "W8", group), (rows, cols)) * std
    scale = (np.max(np.abs(W), axis=0) / 127.0).astype(np.float32)
    q = np.clip(np.rint(W / scale.astype(np.float64)[None, :]), -127, 127).astype(np.int8)
    return q, scale


def mlp_up_w8(seed: int = 1, tokens: int = 4096, hidden: int = 4096, ffn: int = 14336) -> MatmulInputs:
    """MLP up/gate projection with an int8 weight: X as in ``mlp_up`` (bf16) and
    W [hidden x ffn] int8 with per-column scales (``weight_int8``), which are
    kept in ``meta["b_scale"]``."""
    X = llm_activation_bf16(seed, tokens, hidden)
    q, scale = weight_int8(seed, hidden, ffn)
    return MatmulInputs(f"MLP up/gate projection {tokens}x{hidden}x{ffn} bf16 x int8", "bf16", X, q,
                        (0.5,), seed, meta={"b_scale": scale})


@dataclass
class AttentionInputs:
    """Q [B,Hq,S,D], K/V [B,Hkv,S,D] as bf16 bits (row-major, contiguous)."""
    name: str
    Q: np.ndarray
    K: np.ndarray
    V: np.ndarray
    rho_d: float
    rho_t: float
    seed: int
    attempts: list = field(default_factory=list)

    @property
    def shape(self):
        B, Hq, S, D = self.Q.shape
        return B, Hq, self.K.shape[1], S, D


def attention_group(seed: int, B: int, Hq: int, Hkv: int, S: int, D: int, g: int, attempt: int = 0):
    """Draw Q (the Hq/Hkv query heads of kv-group g), K and V (kv head g) for all
    batches: N(0,1) times a per-(head, dim) lognormal(0, 0.5) scale.
    Returns fp64 arrays (unrounded) Qg [B,G,S,D], Kg [B,S,D], Vg [B,S,D]."""
    G = Hq // Hkv
    qs = np.exp(0.5 * _normal(substream(seed, "qscale", g, attempt), (G, D)))
    ks = np.exp(0.5 * _normal(substream(seed, "kscale", g, attempt), D))
    vs = np.exp(0.5 * _normal(substream(seed, "vscale", g, attempt), D))
    Qg = _normal(substream(seed, "Q", g, attempt), (B, G, S, D)) * qs[None, :, None, :]
    Kg = _normal(substream(seed, "K", g, attempt), (B, S, D)) * ks[None, None, :]
    Vg = _normal(substream(seed, "V", g, attempt), (B, S, D)) * vs[None, None, :]
    return Qg, Kg, Vg


def attention(seed: int = 3, B: int = 1, Hq: int = 32, Hkv: int = 32, S: int = 8192, D: int = 128,
              rho_d: float = 0.5, rho_t: float = 0.5, attempts=None) -> AttentionInputs:
    """Attention reduction workload (causal).  ``attempts[g]`` selects the
    redraw attempt of kv-group g (default 0 for every group)."""
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    G = Hq // Hkv
    attempts = list(attempts) if attempts is not None else [0] * Hkv
    Q = np.empty((B, Hq, S, D), np.uint16)
    K = np.empty((B, Hkv, S, D), np.uint16)
    V = np.empty((B, Hkv, S, D), np.uint16)
    for g in range(Hkv):
        Qg, Kg, Vg = attention_group(seed, B, Hq, Hkv, S, D, g, attempts[g])
        Q[:, g * G:(g + 1) * G] = f32_to_bf16_bits(Qg)
        K[:, g] = f32_to_bf16_bits(Kg)
        V[:, g] = f32_to_bf16_bits(Vg)
    name = f"reduced attention B{B} Hq{Hq} Hkv{Hkv} S{S} D{D}"
    return AttentionInputs(name, Q, K, V, rho_d, rho_t, seed, attempts)


@dataclass
class DecodeAttentionInputs:
    """One new query token per sequence over a KV cache: q [B,Hq,D] and caches
    K/V [B,Hkv,Lmax,D] (bf16 bits, contiguous) holding L valid tokens."""
    name: str
    q: np.ndarray
    K: np.ndarray
    V: np.ndarray
    L: int
    rho_d: float
    rho_t: float
    seed: int
    attempts: list = field(default_factory=list)

    @property
    def shape(self):
        B, Hq, D = self.q.shape
        return B, Hq, self.K.shape[1], self.L, self.K.shape[2], D


def decode_attention(seed: int = 5, B: int = 1, Hq: int = 32, Hkv: int = 8, L: int = 32768, D: int = 128,
                     rho_d: float = 0.5, rho_t: float = 0.5, Lmax: int = None, attempts=None) -> DecodeAttentionInputs:
    """Decode-step workload: per kv-group g, q (its Hq/Hkv heads), K and V drawn
    as N(0,1) times a per-(head, dim) lognormal(0, 0.5) scale, as in the
    prefill workload.  Cache rows L..Lmax-1 (unused capacity) hold 1e4, so a
    read past the valid length would show.  ``attempts[g]`` selects the
    redraw attempt of kv-group g."""
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    Lmax = L if Lmax is None else Lmax
    if not (1 <= L <= Lmax):
        raise ValueError("need 1 <= L <= Lmax")
    G = Hq // Hkv
    attempts = list(attempts) if attempts is not None else [0] * Hkv
    q = np.empty((B, Hq, D), np.uint16)
    K = np.full((B, Hkv, Lmax, D), f32_to_bf16_bits(np.float32(1e4)), np.uint16)
    V = np.full((B, Hkv, Lmax, D), f32_to_bf16_bits(np.float32(1e4)), np.uint16)
    for g in range(Hkv):
        a = attempts[g]
        qs = np.exp(0.5 * _normal(substream(seed, "qscale", g, a), (G, D)))
        ks = np.exp(0.5 * _normal(substream(seed, "kscale", g, a), D))
        vs = np.exp(0.5 * _normal(substream(seed, "vscale", g, a), D))
        q[:, g * G:(g + 1) * G] = f32_to_bf16_bits(_normal(substream(seed, "Q", g, a), (B, G, D)) * qs[None])
        K[:, g, :L] = f32_to_bf16_bits(_normal(substream(seed, "K", g, a), (B, L, D)) * ks[None, None, :])
        V[:, g, :L] = f32_to_bf16_bits(_normal(substream(seed, "V", g, a), (B, L, D)) * vs[None, None, :])
    return DecodeAttentionInputs(f"decode attention B{B} Hq{Hq} Hkv{Hkv} L{L} D{D}", q, K, V, L, rho_d, rho_t,
                                 seed, attempts)
