"""Python binding of librmm (Reduced Matrix Multiplication on B200, sm_100a).

Argument marshalling only: every step of the path runs in the CUDA kernels of
``librmm.so`` behind the C ABI declared in ``include/rmm.h``.  PyTorch is used
for device memory and streams.  There is no fallback: importing this package
without the built library raises, and every call whose status is not RMM_OK
raises ``RMMError``.

The functions keep the C names (``rmm_score``, ``rmm_topk``, ``rmm_compact``,
``rmm_gemm``, ``rmm_matmul``, ``rmm_attention`` ...) and take torch tensors;
``lib`` is the raw ctypes handle for pointer-level calls.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

__all__ = [
    "lib", "LIB_PATH", "RMMError", "RMM_F32", "RMM_BF16", "rmm_abi_version", "rmm_k_from_rho",
    "rmm_device_error", "rmm_score", "rmm_score_workspace_size", "rmm_score_noalloc", "rmm_topk", "rmm_compact", "rmm_gather_rows", "rmm_compact_gather",
    "rmm_gemm", "rmm_gemm_workspace_size", "rmm_gemm_compacted",
    "rmm_matmul", "rmm_matmul_workspace_size", "rmm_gemm_w8", "rmm_gemm_w8_workspace_size", "rmm_matmul_w8",
    "rmm_matmul_w8_workspace_size", "rmm_attention", "rmm_attention_workspace_size", "rmm_decode_attention",
    "rmm_decode_attention_workspace_size", "rmm_matmul_multi", "rmm_matmul_multi_workspace_size",
    "rmm_silu_mul_score", "rmm_silu_mul_score_workspace_size", "rmm_mlp_block", "rmm_mlp_block_workspace_size",
    "rmm_selftest_timeout", "exported_symbols", "declared_symbols",
]

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT_DIR = os.path.dirname(PKG_DIR)
LIB_PATH = os.path.join(PKG_DIR, "librmm.so")
HEADER_PATH = os.path.join(ROOT_DIR, "include", "rmm.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"librmm.so not built ({LIB_PATH}); run: python input_adaptive_reduced_score_b200/build.py")

lib = ctypes.CDLL(LIB_PATH)

RMM_F32, RMM_BF16 = 0, 1
_STATUS = {0: "RMM_OK", 1: "RMM_ERR_INVALID_ARG", 2: "RMM_ERR_UNSUPPORTED", 3: "RMM_ERR_WORKSPACE",
           4: "RMM_ERR_CUDA", 5: "RMM_ERR_DEVICE"}

c_i64, c_int, c_sz, c_dbl, c_flt, c_vp = (ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_double,
                                          ctypes.c_float, ctypes.c_void_p)


def _sig(name, res, *args):
    try:
        f = getattr(lib, name)
    except AttributeError:
        raise ImportError(f"{LIB_PATH} does not export {name} (built from older sources?); "
                          "run: python input_adaptive_reduced_score_b200/build.py") from None
    f.restype = res
    f.argtypes = list(args)
    return f


_sig("rmm_abi_version", c_int)
_sig("rmm_last_error", ctypes.c_char_p)
_sig("rmm_k_from_rho", c_i64, c_dbl, c_i64)
_sig("rmm_device_error", c_int, c_vp, c_int, ctypes.POINTER(ctypes.c_uint))
_sig("rmm_score_workspace_size", c_sz, c_int, c_i64, c_i64, c_i64)
_sig("rmm_score", c_int, c_vp, c_int, c_i64, c_i64, c_i64, c_i64, c_i64, c_vp, c_i64, c_int, c_vp, c_sz, c_vp)
_sig("rmm_score_noalloc", c_int, c_vp, c_int, c_i64, c_i64, c_i64, c_i64, c_i64, c_vp, c_i64, c_int, c_vp)
_sig("rmm_topk", c_int, c_vp, c_i64, c_i64, c_i64, c_i64, c_vp, c_i64, c_vp)
_sig("rmm_compact", c_int, c_vp, c_int, c_i64, c_i64, c_i64, c_vp, c_i64, c_vp, c_i64, c_vp)
_sig("rmm_gather_rows", c_int, c_vp, c_int, c_i64, c_i64, c_i64, c_vp, c_i64, c_vp, c_i64, c_vp)
_sig("rmm_compact_gather", c_int, c_vp, c_i64, c_vp, c_i64, c_i64, c_i64, c_i64, c_vp, c_i64, c_vp, c_i64, c_vp, c_i64,
     c_vp)
_sig("rmm_gemm_workspace_size", c_sz, c_int, c_i64, c_i64)
_sig("rmm_gemm", c_int, c_vp, c_i64, c_vp, c_i64, c_vp, c_i64, c_i64, c_i64, c_i64, c_int, c_vp, c_int, c_i64, c_vp,
     c_sz, c_vp)
_sig("rmm_gemm_compacted", c_int, c_vp, c_i64, c_vp, c_i64, c_i64, c_i64, c_i64, c_vp, c_int, c_i64, c_vp)
_sig("rmm_matmul_workspace_size", c_sz, c_int, c_i64, c_i64, c_i64, c_dbl)
_sig("rmm_matmul", c_int, c_vp, c_i64, c_vp, c_i64, c_i64, c_i64, c_i64, c_dbl, c_int, c_vp, c_int, c_i64, c_vp, c_vp,
     c_vp, c_sz, c_vp)
_sig("rmm_gemm_w8_workspace_size", c_sz, c_i64, c_i64)
_sig("rmm_gemm_w8", c_int, c_vp, c_i64, c_vp, c_i64, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_vp, c_int, c_i64, c_vp,
     c_sz, c_vp)
_sig("rmm_matmul_w8_workspace_size", c_sz, c_i64, c_i64, c_i64, c_dbl)
_sig("rmm_matmul_w8", c_int, c_vp, c_i64, c_vp, c_i64, c_vp, c_i64, c_i64, c_i64, c_dbl, c_vp, c_int, c_i64, c_vp, c_vp,
     c_vp, c_sz, c_vp)
_sig("rmm_decode_attention_workspace_size", c_sz, c_i64, c_i64, c_i64, c_i64, c_dbl, c_int, c_int)
_sig("rmm_decode_attention", c_int, c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_i64, c_i64, c_dbl, c_dbl, c_flt,
     c_vp, c_int, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp)
_sig("rmm_matmul_multi_workspace_size", c_sz, c_i64, c_i64, c_i64, c_dbl)
_sig("rmm_matmul_multi", c_int, c_vp, c_i64, c_i64, c_i64, c_dbl, c_int, c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_vp,
     c_vp, c_vp, c_vp, c_sz, c_vp)
_sig("rmm_silu_mul_score_workspace_size", c_sz, c_i64, c_i64)
_sig("rmm_silu_mul_score", c_int, c_vp, c_i64, c_vp, c_i64, c_i64, c_i64, c_vp, c_i64, c_vp, c_vp, c_sz, c_vp)
_sig("rmm_mlp_block_workspace_size", c_sz, c_i64, c_i64, c_i64, c_dbl, c_dbl)
_sig("rmm_mlp_block", c_int, c_vp, c_i64, c_i64, c_i64, c_i64, c_vp, c_i64, c_vp, c_i64, c_vp, c_i64, c_dbl, c_dbl,
     c_vp, c_int, c_i64, c_vp, c_vp, c_vp, c_sz, c_vp)
_sig("rmm_attention_workspace_size", c_sz, c_i64, c_i64, c_i64, c_i64, c_i64, c_dbl, c_dbl)
_sig("rmm_attention", c_int, c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_i64, c_dbl, c_dbl, c_flt, c_vp, c_int,
     c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp)
_sig("rmm_selftest_timeout", c_int, c_int, c_vp)


class RMMError(RuntimeError):
    def __init__(self, status, where):
        msg = lib.rmm_last_error().decode(errors="replace")
        super().__init__(f"{where}: {_STATUS.get(status, status)}: {msg}")
        self.status = status


def _check(status, where):
    if status != 0:
        raise RMMError(status, where)


def declared_symbols():
    """Function names declared with RMM_API in include/rmm.h."""
    with open(HEADER_PATH) as f:
        return sorted(set(re.findall(r"^RMM_API\s+[\w\s\*]+?\b(rmm_\w+)\s*\(", f.read(), re.M)))


def exported_symbols():
    return [s for s in declared_symbols() if hasattr(lib, s)]


# ------------------------------------------------------------------ helpers

def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return RMM_BF16
    if t.dtype == torch.float32:
        return RMM_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream_ptr(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return c_vp(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t):
    return c_vp(0 if t is None else t.data_ptr())


def _row_major(t: torch.Tensor, name: str):
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D row-major tensor (unit column stride)")
    return t.stride(0)


def _workspace(nbytes: int, device, ws):
    if nbytes == 0:
        return None, 0
    if ws is not None:
        if ws.numel() * ws.element_size() < nbytes:
            raise ValueError(f"workspace too small: need {nbytes} bytes")
        return ws, ws.numel() * ws.element_size()
    return torch.empty(nbytes, dtype=torch.uint8, device=device), nbytes


# ------------------------------------------------------------------ API

def rmm_abi_version() -> int:
    return lib.rmm_abi_version()


def rmm_k_from_rho(rho: float, d: int) -> int:
    return lib.rmm_k_from_rho(float(rho), int(d))


def rmm_device_error(stream=None, clear: bool = True) -> int:
    """Synchronise the stream and return the device error word (0 = none)."""
    code = ctypes.c_uint(0)
    st = lib.rmm_device_error(_stream_ptr(stream), int(clear), ctypes.byref(code))
    if st not in (0, 5):
        _check(st, "rmm_device_error")
    return code.value


def rmm_selftest_timeout(which: int, stream=None) -> int:
    """Make one of the library's bounded waits run out on purpose (0: an
    mbarrier nothing arrives on; 1: a flag nothing raises; 2: the CTA-pair
    product whose row copy never runs) and return the device error word it
    left (RMM_DEVERR_TIMEOUT_BASE + site), clearing it.  Takes about 2 s."""
    _check(lib.rmm_selftest_timeout(int(which), _stream_ptr(stream)), "rmm_selftest_timeout")
    return rmm_device_error(stream, clear=True)


def rmm_score_workspace_size(dtype: int, batch: int, M: int, d: int) -> int:
    return lib.rmm_score_workspace_size(dtype, batch, M, d)


def rmm_score(A: torch.Tensor, out: torch.Tensor = None, sqrt_out: bool = False, ws=None, stream=None):
    """Column scores ss_j = sum_i A[i,j]^2 of A [M x d] or a batch A [b x M x d]."""
    batched = A.dim() == 3
    A3 = A if batched else A.unsqueeze(0)
    if A3.stride(2) != 1:
        raise ValueError("A must have unit column stride")
    b, M, d = A3.shape
    dt = _dtype_code(A3)
    if out is None:
        out = torch.empty((b, d), dtype=torch.float32, device=A.device)
    out2 = out if out.dim() == 2 else out.view(1, -1)
    wsb = lib.rmm_score_workspace_size(dt, b, M, d)
    w, wn = _workspace(wsb, A.device, ws)
    _check(lib.rmm_score(_ptr(A3), dt, b, M, d, A3.stride(1), A3.stride(0) if b > 1 else 0, _ptr(out2),
                         out2.stride(0), int(sqrt_out), _ptr(w), wn, _stream_ptr(stream)), "rmm_score")
    return out if batched or out.dim() == 1 else out2[0]


def rmm_score_noalloc(A: torch.Tensor, out: torch.Tensor = None, sqrt_out: bool = False, stream=None):
    """rmm_score without a workspace argument: the partial sums use the
    library's built-in scratch array (for callers that cannot allocate)."""
    batched = A.dim() == 3
    A3 = A if batched else A.unsqueeze(0)
    if A3.stride(2) != 1:
        raise ValueError("A must have unit column stride")
    b, M, d = A3.shape
    if out is None:
        out = torch.empty((b, d), dtype=torch.float32, device=A.device)
    out2 = out if out.dim() == 2 else out.view(1, -1)
    _check(lib.rmm_score_noalloc(_ptr(A3), _dtype_code(A3), b, M, d, A3.stride(1), A3.stride(0) if b > 1 else 0,
                                 _ptr(out2), out2.stride(0), int(sqrt_out), _stream_ptr(stream)),
           "rmm_score_noalloc")
    return out if batched or out.dim() == 1 else out2[0]


def rmm_topk(scores: torch.Tensor, k: int, out: torch.Tensor = None, stream=None):
    """Ascending top-k indices (int32) per row of scores [d] or [b x d]."""
    s2 = scores if scores.dim() == 2 else scores.view(1, -1)
    if s2.dtype != torch.float32 or s2.stride(1) != 1:
        raise ValueError("scores must be fp32 with unit stride")
    b, d = s2.shape
    if out is None:
        out = torch.empty((b, k), dtype=torch.int32, device=scores.device)
    o2 = out if out.dim() == 2 else out.view(1, -1)
    _check(lib.rmm_topk(_ptr(s2), b, d, s2.stride(0), k, _ptr(o2), o2.stride(0), _stream_ptr(stream)), "rmm_topk")
    return out if scores.dim() == 2 else o2[0]


def rmm_compact(A: torch.Tensor, idx: torch.Tensor, out: torch.Tensor = None, stream=None):
    """A_I[:, r] = A[:, idx[r]] for A [M x d]."""
    lda = _row_major(A, "A")
    M, d = A.shape
    k = idx.numel()
    if out is None:
        ld = (k + 7) // 8 * 8
        out = torch.empty((M, ld), dtype=A.dtype, device=A.device)[:, :k]
    _check(lib.rmm_compact(_ptr(A), _dtype_code(A), M, d, lda, _ptr(idx), k, _ptr(out), out.stride(0),
                           _stream_ptr(stream)), "rmm_compact")
    return out


def rmm_gather_rows(B: torch.Tensor, idx: torch.Tensor, out: torch.Tensor = None, stream=None):
    """B_I[r, :] = B[idx[r], :] for B [d x N]."""
    ldb = _row_major(B, "B")
    d, N = B.shape
    k = idx.numel()
    if out is None:
        ld = (N + 7) // 8 * 8
        out = torch.empty((k, ld), dtype=B.dtype, device=B.device)[:, :N]
    _check(lib.rmm_gather_rows(_ptr(B), _dtype_code(B), d, N, ldb, _ptr(idx), k, _ptr(out), out.stride(0),
                               _stream_ptr(stream)), "rmm_gather_rows")
    return out


def rmm_compact_gather(A: torch.Tensor, B: torch.Tensor, idx: torch.Tensor, out_a: torch.Tensor = None,
                       out_b: torch.Tensor = None, stream=None):
    """A_I = A[:, idx] and B_I = B[idx, :] in one launch (bf16); returns (A_I, B_I)."""
    lda = _row_major(A, "A")
    ldb = _row_major(B, "B")
    M, d = A.shape
    if B.shape[0] != d:
        raise ValueError("A and B disagree on d")
    N = B.shape[1]
    k = idx.numel()
    if out_a is None:
        out_a = torch.empty((M, (k + 7) // 8 * 8), dtype=A.dtype, device=A.device)[:, :k]
    if out_b is None:
        out_b = torch.empty((k, (N + 7) // 8 * 8), dtype=B.dtype, device=B.device)[:, :N]
    if A.dtype != torch.bfloat16 or B.dtype != torch.bfloat16:
        raise TypeError("rmm_compact_gather takes bf16 operands")
    _check(lib.rmm_compact_gather(_ptr(A), lda, _ptr(B), ldb, M, d, N, _ptr(idx), k, _ptr(out_a), out_a.stride(0),
                                  _ptr(out_b), out_b.stride(0), _stream_ptr(stream)), "rmm_compact_gather")
    return out_a, out_b


def rmm_gemm_workspace_size(dtype: int, N: int, k: int) -> int:
    return lib.rmm_gemm_workspace_size(dtype, N, k)


def rmm_gemm(A_I: torch.Tensor, B: torch.Tensor, idx: torch.Tensor, out: torch.Tensor = None,
             out_dtype=None, ws=None, stream=None):
    """Y = A_I · B[idx, :], A_I [M x k] (compacted), B [d x N]."""
    ld_ai = _row_major(A_I, "A_I")
    ldb = _row_major(B, "B")
    M, k = A_I.shape
    d, N = B.shape
    if idx.numel() != k:
        raise ValueError("idx must hold k indices")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype or A_I.dtype, device=A_I.device)
    ldy = _row_major(out, "Y")
    dt = _dtype_code(A_I)
    w, wn = _workspace(lib.rmm_gemm_workspace_size(dt, N, k), A_I.device, ws)
    _check(lib.rmm_gemm(_ptr(A_I), ld_ai, _ptr(B), ldb, _ptr(idx), d, M, N, k, dt, _ptr(out),
                        _dtype_code(out), ldy, _ptr(w), wn, _stream_ptr(stream)), "rmm_gemm")
    return out


def rmm_gemm_compacted(A_I: torch.Tensor, B_I: torch.Tensor, out: torch.Tensor = None, out_dtype=None,
                       stream=None):
    """Y = A_I · B_I on compacted bf16 operands A_I [M x k], B_I [k x N]."""
    ld_ai = _row_major(A_I, "A_I")
    ld_bi = _row_major(B_I, "B_I")
    M, k = A_I.shape
    N = B_I.shape[1]
    if B_I.shape[0] != k:
        raise ValueError("A_I and B_I disagree on k")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype or A_I.dtype, device=A_I.device)
    ldy = _row_major(out, "Y")
    _check(lib.rmm_gemm_compacted(_ptr(A_I), ld_ai, _ptr(B_I), ld_bi, M, N, k, _ptr(out), _dtype_code(out), ldy,
                                  _stream_ptr(stream)), "rmm_gemm_compacted")
    return out


def rmm_matmul_workspace_size(dtype: int, M: int, d: int, N: int, rho: float) -> int:
    return lib.rmm_matmul_workspace_size(dtype, M, d, N, float(rho))


def rmm_matmul(A: torch.Tensor, B: torch.Tensor, rho: float, out: torch.Tensor = None, out_dtype=None,
               idx_out: torch.Tensor = None, ss_out: torch.Tensor = None, ws=None, stream=None):
    """The whole path: score -> top-k -> compaction -> reduced GEMM."""
    lda = _row_major(A, "A")
    ldb = _row_major(B, "B")
    M, d = A.shape
    N = B.shape[1]
    dt = _dtype_code(A)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype or A.dtype, device=A.device)
    ldy = _row_major(out, "Y")
    wsb = lib.rmm_matmul_workspace_size(dt, M, d, N, float(rho))
    w, wn = _workspace(wsb, A.device, ws)
    _check(lib.rmm_matmul(_ptr(A), lda, _ptr(B), ldb, M, d, N, float(rho), dt, _ptr(out), _dtype_code(out), ldy,
                          _ptr(idx_out), _ptr(ss_out), _ptr(w), wn, _stream_ptr(stream)), "rmm_matmul")
    return out


def _int8_weight(Bq: torch.Tensor, b_scale: torch.Tensor):
    if Bq.dtype != torch.int8:
        raise TypeError("Bq must be int8")
    if b_scale.dtype != torch.float32 or b_scale.numel() != Bq.shape[1] or not b_scale.is_contiguous():
        raise ValueError("b_scale must be a contiguous fp32 vector of N column scales")
    return _row_major(Bq, "Bq")


def rmm_gemm_w8_workspace_size(N: int, k: int) -> int:
    return lib.rmm_gemm_w8_workspace_size(N, k)


def rmm_gemm_w8(A_I: torch.Tensor, Bq: torch.Tensor, b_scale: torch.Tensor, idx: torch.Tensor,
                out: torch.Tensor = None, out_dtype=None, ws=None, stream=None):
    """Y = A_I · (Bq[idx, :] * b_scale), A_I bf16 [M x k], Bq int8 [d x N], b_scale fp32 [N]."""
    ld_ai = _row_major(A_I, "A_I")
    ldb = _int8_weight(Bq, b_scale)
    M, k = A_I.shape
    d, N = Bq.shape
    if idx.numel() != k:
        raise ValueError("idx must hold k indices")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype or A_I.dtype, device=A_I.device)
    ldy = _row_major(out, "Y")
    w, wn = _workspace(lib.rmm_gemm_w8_workspace_size(N, k), A_I.device, ws)
    _check(lib.rmm_gemm_w8(_ptr(A_I), ld_ai, _ptr(Bq), ldb, _ptr(b_scale), _ptr(idx), d, M, N, k, _ptr(out),
                           _dtype_code(out), ldy, _ptr(w), wn, _stream_ptr(stream)), "rmm_gemm_w8")
    return out


def rmm_matmul_w8_workspace_size(M: int, d: int, N: int, rho: float) -> int:
    return lib.rmm_matmul_w8_workspace_size(M, d, N, float(rho))


def rmm_matmul_w8(A: torch.Tensor, Bq: torch.Tensor, b_scale: torch.Tensor, rho: float, out: torch.Tensor = None,
                  out_dtype=None, idx_out: torch.Tensor = None, ss_out: torch.Tensor = None, ws=None, stream=None):
    """The whole path with an int8 weight: score -> top-k -> compaction -> reduced product."""
    lda = _row_major(A, "A")
    ldb = _int8_weight(Bq, b_scale)
    M, d = A.shape
    N = Bq.shape[1]
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype or A.dtype, device=A.device)
    ldy = _row_major(out, "Y")
    w, wn = _workspace(lib.rmm_matmul_w8_workspace_size(M, d, N, float(rho)), A.device, ws)
    _check(lib.rmm_matmul_w8(_ptr(A), lda, _ptr(Bq), ldb, _ptr(b_scale), M, d, N, float(rho), _ptr(out),
                             _dtype_code(out), ldy, _ptr(idx_out), _ptr(ss_out), _ptr(w), wn, _stream_ptr(stream)),
           "rmm_matmul_w8")
    return out


def rmm_attention_workspace_size(B, Hq, Hkv, S, D, rho_d, rho_t) -> int:
    return lib.rmm_attention_workspace_size(B, Hq, Hkv, S, D, float(rho_d), float(rho_t))


def rmm_attention(Q, K, V, rho_d: float, rho_t: float, scale: float = 0.0, out=None, out_dtype=None,
                  idx_d=None, idx_t=None, lse=None, tscore=None, ws=None, stream=None):
    """Reduced causal attention; Q [B,Hq,S,D], K/V [B,Hkv,S,D] bf16 contiguous."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{n} must be a contiguous 4-D bf16 tensor")
    B, Hq, S, D = Q.shape
    Hkv = K.shape[1]
    if out is None:
        out = torch.empty((B, Hq, S, D), dtype=out_dtype or torch.bfloat16, device=Q.device)
    wsb = lib.rmm_attention_workspace_size(B, Hq, Hkv, S, D, float(rho_d), float(rho_t))
    w, wn = _workspace(wsb, Q.device, ws)
    _check(lib.rmm_attention(_ptr(Q), _ptr(K), _ptr(V), B, Hq, Hkv, S, D, float(rho_d), float(rho_t), float(scale),
                             _ptr(out), _dtype_code(out), _ptr(idx_d), _ptr(idx_t), _ptr(lse), _ptr(tscore),
                             _ptr(w), wn, _stream_ptr(stream)), "rmm_attention")
    return out


def rmm_decode_attention_workspace_size(B, Hq, L, D, rho_t, with_logits=False, with_idx_t=False) -> int:
    return lib.rmm_decode_attention_workspace_size(B, Hq, L, D, float(rho_t), int(bool(with_logits)),
                                                   int(bool(with_idx_t)))


def rmm_decode_attention(q, K, V, L: int, rho_d: float, rho_t: float, scale: float = 0.0, out=None, out_dtype=None,
                         idx_d=None, idx_t=None, lse=None, logits=None, ws=None, stream=None):
    """Reduced attention of one new query token per sequence over a KV cache:
    q [B,Hq,D], caches K/V [B,Hkv,Lmax,D] (bf16, contiguous) holding L tokens."""
    if q.dtype != torch.bfloat16 or not q.is_contiguous() or q.dim() != 3:
        raise ValueError("q must be a contiguous [B, Hq, D] bf16 tensor")
    for t, n in ((K, "K"), (V, "V")):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{n} must be a contiguous [B, Hkv, Lmax, D] bf16 tensor")
    B, Hq, D = q.shape
    Hkv, Lmax = K.shape[1], K.shape[2]
    if out is None:
        out = torch.empty((B, Hq, D), dtype=out_dtype or torch.bfloat16, device=q.device)
    wsb = lib.rmm_decode_attention_workspace_size(B, Hq, L, D, float(rho_t), int(logits is not None),
                                                  int(idx_t is not None))
    w, wn = _workspace(wsb, q.device, ws)
    _check(lib.rmm_decode_attention(_ptr(q), _ptr(K), _ptr(V), B, Hq, Hkv, L, Lmax, D, float(rho_d), float(rho_t),
                                    float(scale), _ptr(out), _dtype_code(out), _ptr(idx_d), _ptr(idx_t), _ptr(lse),
                                    _ptr(logits), _ptr(w), wn, _stream_ptr(stream)), "rmm_decode_attention")
    return out


def rmm_matmul_multi_workspace_size(M: int, d: int, N_max: int, rho: float) -> int:
    return lib.rmm_matmul_multi_workspace_size(M, d, N_max, float(rho))


def rmm_matmul_multi(A: torch.Tensor, Bs, rho: float, outs=None, out_dtype=None, ss_in: torch.Tensor = None,
                     idx_out: torch.Tensor = None, ss_out: torch.Tensor = None, ws=None, stream=None):
    """Y[i] = A[:, I] @ Bs[i][I, :] with one selection I shared by every weight."""
    lda = _row_major(A, "A")
    M, d = A.shape
    n = len(Bs)
    if outs is None:
        outs = [torch.empty((M, B.shape[1]), dtype=out_dtype or A.dtype, device=A.device) for B in Bs]
    ldb = [_row_major(B, "B") for B in Bs]
    ldy = [_row_major(Y, "Y") for Y in outs]
    Ns = [B.shape[1] for B in Bs]
    arr_p = (ctypes.c_void_p * n)(*[_ptr(B) for B in Bs])
    arr_y = (ctypes.c_void_p * n)(*[_ptr(Y) for Y in outs])
    arr_ldb = (ctypes.c_int64 * n)(*ldb)
    arr_n = (ctypes.c_int64 * n)(*Ns)
    arr_ldy = (ctypes.c_int64 * n)(*ldy)
    w, wn = _workspace(lib.rmm_matmul_multi_workspace_size(M, d, max(Ns), float(rho)), A.device, ws)
    _check(lib.rmm_matmul_multi(_ptr(A), lda, M, d, float(rho), n, ctypes.cast(arr_p, c_vp), ctypes.cast(arr_ldb, c_vp),
                                ctypes.cast(arr_n, c_vp), ctypes.cast(arr_y, c_vp), ctypes.cast(arr_ldy, c_vp),
                                _dtype_code(outs[0]), _ptr(ss_in), _ptr(idx_out), _ptr(ss_out), _ptr(w), wn,
                                _stream_ptr(stream)), "rmm_matmul_multi")
    return outs


def rmm_silu_mul_score_workspace_size(M: int, N: int) -> int:
    return lib.rmm_silu_mul_score_workspace_size(M, N)


def rmm_silu_mul_score(G: torch.Tensor, U: torch.Tensor, out: torch.Tensor = None, ss_out: torch.Tensor = None,
                       ws=None, stream=None):
    """H = bf16(SiLU(G) * U) and the column scores of H in one pass; returns (H, ss)."""
    ldg, ldu = _row_major(G, "G"), _row_major(U, "U")
    M, N = G.shape
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=G.device)
    if ss_out is None:
        ss_out = torch.empty(N, dtype=torch.float32, device=G.device)
    w, wn = _workspace(lib.rmm_silu_mul_score_workspace_size(M, N), G.device, ws)
    _check(lib.rmm_silu_mul_score(_ptr(G), ldg, _ptr(U), ldu, M, N, _ptr(out), _row_major(out, "H"), _ptr(ss_out),
                                  _ptr(w), wn, _stream_ptr(stream)), "rmm_silu_mul_score")
    return out, ss_out


def rmm_mlp_block_workspace_size(M: int, d_model: int, d_ff: int, rho_up: float, rho_down: float) -> int:
    return lib.rmm_mlp_block_workspace_size(M, d_model, d_ff, float(rho_up), float(rho_down))


def rmm_mlp_block(X: torch.Tensor, W_up: torch.Tensor, W_gate: torch.Tensor, W_down: torch.Tensor, rho_up: float,
                  rho_down: float, out: torch.Tensor = None, out_dtype=None, idx_up: torch.Tensor = None,
                  idx_down: torch.Tensor = None, ws=None, stream=None):
    """Gated MLP block, every product reduced: Y = RMM(SiLU(RMM(X, W_gate)) * RMM(X, W_up), W_down)."""
    ldx = _row_major(X, "X")
    M, d_model = X.shape
    d_ff = W_up.shape[1]
    if out is None:
        out = torch.empty((M, d_model), dtype=out_dtype or X.dtype, device=X.device)
    w, wn = _workspace(lib.rmm_mlp_block_workspace_size(M, d_model, d_ff, float(rho_up), float(rho_down)),
                       X.device, ws)
    _check(lib.rmm_mlp_block(_ptr(X), ldx, M, d_model, d_ff, _ptr(W_up), _row_major(W_up, "W_up"), _ptr(W_gate),
                             _row_major(W_gate, "W_gate"), _ptr(W_down), _row_major(W_down, "W_down"),
                             float(rho_up), float(rho_down), _ptr(out), _dtype_code(out), _row_major(out, "Y"),
                             _ptr(idx_up), _ptr(idx_down), _ptr(w), wn, _stream_ptr(stream)), "rmm_mlp_block")
    return out
