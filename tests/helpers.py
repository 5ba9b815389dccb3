"""Shared test helpers: moving generated inputs to the device and error metrics.
Holds none of the method's arithmetic."""
import numpy as np
import torch


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> torch.bfloat16 tensor (bit-exact)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def to_device(x: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    if dtype == "bf16":
        return bf16_tensor(x, device)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def rel_fro(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def sample_rows(M: int, n: int = 96, seed: int = 0, block: int = 128) -> np.ndarray:
    """Rows spread over every 128-row block (plus the first and last row)."""
    rng = np.random.default_rng(seed)
    rows = {0, M - 1}
    nb = (M + block - 1) // block
    for b in range(nb):
        lo, hi = b * block, min(M, (b + 1) * block)
        rows.add(int(rng.integers(lo, hi)))
    extra = rng.integers(0, M, size=max(0, n - len(rows)))
    rows.update(int(r) for r in extra)
    return np.array(sorted(rows))


def bf16_ulp(x) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def check_bf16_output(got, ref, absprod=None, k=None, fro_tol=2e-3, min_stat=4096):
    """bf16-stored result vs the fp64 oracle.

    Elementwise: |got - ref| <= one bf16 ulp of |ref| (the single rounding of
    the fp32 accumulator) + k * 2^-24 * sum_i |a_i b_i| (the worst-case error of
    an fp32 sum of k exact products, any order), where `absprod` holds
    sum_i |a_i b_i| per element.  Relative Frobenius error <= fro_tol when the
    output has at least `min_stat` elements, and always <= 2^-8 (rounding to 8
    significant bits) plus slack."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    bound = bf16_ulp(np.maximum(np.abs(got), np.abs(ref))) + 1e-30
    if absprod is not None:
        bound = bound + k * 2.0 ** -24 * np.asarray(absprod, dtype=np.float64)
    bad = np.abs(got - ref) > bound
    assert not bad.any(), f"{bad.sum()} elements beyond the bound, e.g. {got[bad][:4]} vs {ref[bad][:4]}"
    err = rel_fro(got, ref)
    limit = fro_tol if got.size >= min_stat else 2.0 ** -8 + 1e-4
    assert err <= limit, (err, limit)
    return err
