"""Failure detection on the GPU without a GPU fault: the library's bounded
waits are made to run out on purpose (an mbarrier nothing arrives on, a flag
nothing raises, and the CTA-pair product whose row copy never runs).  Each
must give up after its limit (2 s), leave RMM_DEVERR_TIMEOUT_BASE + its site
in the device error word, and let its kernel return, so that the context
stays usable: a product right after is checked against the oracle."""
import time

import pytest
import torch

import oracle
import workloads as W
from oracle.conditioning import widen_topk_gaps
from tests.helpers import bf16_tensor, rel_fro, to_f64

pytestmark = pytest.mark.gpu
R = None

TIMEOUT_BASE = 0x100


@pytest.fixture(autouse=True, scope="module")
def _lib():
    global R
    import input_adaptive_reduced_score_b200 as mod
    R = mod
    assert R.rmm_device_error(clear=True) == 0


def _product_still_correct():
    d, rho = 512, 0.5
    inp = W.scaled_matmul_bf16(7, 300, d, 264)
    cond, _ = widen_topk_gaps(inp.A, "bf16", [oracle.k_from_rho(rho, d)])
    Ac = oracle.decode(cond, "bf16")
    Bm = oracle.decode(inp.B, "bf16")
    Y = R.rmm_matmul(bf16_tensor(cond), bf16_tensor(inp.B), rho, out_dtype=torch.float32)
    ref, _, _ = oracle.rmm_path(Ac, Bm, rho)
    assert R.rmm_device_error(clear=True) == 0
    assert rel_fro(to_f64(Y), ref) <= 1e-5


@pytest.mark.parametrize("which,sites", [(0, {62}), (1, {63}), (2, {43, 44, 45})])
def test_bounded_wait_runs_out(which, sites):
    t0 = time.monotonic()
    code = R.rmm_selftest_timeout(which)
    elapsed = time.monotonic() - t0
    assert code - TIMEOUT_BASE in sites, hex(code)
    assert 1.5 < elapsed < 30.0, elapsed
    _product_still_correct()
