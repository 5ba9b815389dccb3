"""Host logic of bench.py that needs no GPU: the rho sweep's bookkeeping and
its error isolation (a failing run is recorded in its own entry and the
other entries are still measured), with the library and the CUDA events
replaced by fakes."""
import types

import pytest
import torch

import bench


class _Event:
    def __init__(self, **kw):
        pass

    def record(self, stream=None):
        pass


def _timed(fn, steps, nev):
    for _ in range(steps):
        fn([_Event() for _ in range(nev)])
    return [[0.25] for _ in range(steps)]  # 0.25 ms per step


def _fake_lib(fail_at=None):
    calls = []

    def matmul(A, B, rho, out=None, ws=None):
        calls.append(rho)
        if rho == fail_at:
            raise RuntimeError("planted failure")
    return types.SimpleNamespace(
        RMM_BF16=1,
        rmm_k_from_rho=lambda rho, d: max(1, min(d, int(-(-rho * d // 1)))),
        rmm_matmul_workspace_size=lambda dtype, M, d, N, rho: 256,
        rmm_matmul=matmul,
        rmm_device_error=lambda stream: 0), calls


@pytest.fixture(autouse=True)
def _no_cuda_events(monkeypatch):
    monkeypatch.setattr(torch.cuda, "Event", _Event)


def test_rho_sweep_reports_each_rho():
    R, calls = _fake_lib()
    M, d, N = 64, 40, 16
    A = torch.zeros(M, d, dtype=torch.bfloat16)
    B = torch.zeros(d, N, dtype=torch.bfloat16)
    out = bench.rho_sweep(R, A, B, (0.7, 1.0), 0.5, 4, _timed, None, "cpu")
    assert set(out) == {"rho=0.7", "rho=1.0"}
    for rho, e in ((0.7, out["rho=0.7"]), (1.0, out["rho=1.0"])):
        k = R.rmm_k_from_rho(rho, d)
        assert e["k"] == k
        assert e["step_us"] == pytest.approx(250.0)
        assert e["effective_tflops"] == pytest.approx(2.0 * M * N * k / 0.25e-3 / 1e12)
        assert e["speedup_vs_dense"] == pytest.approx(2.0)
    # three warm-up calls and four timed steps per rho
    assert calls.count(0.7) == 7 and calls.count(1.0) == 7


def test_rho_sweep_isolates_a_failure():
    R, _ = _fake_lib(fail_at=0.8)
    A = torch.zeros(32, 32, dtype=torch.bfloat16)
    B = torch.zeros(32, 8, dtype=torch.bfloat16)
    out = bench.rho_sweep(R, A, B, (0.8, 1.0), 0.5, 2, _timed, None, "cpu")
    assert "planted failure" in out["rho=0.8"]["error"]
    assert out["rho=1.0"]["step_us"] == pytest.approx(250.0)
