"""Failure detection without a GPU fault: a pipeline wait that runs out.

The self-test kernel waits, with the bounded wait every GEMM stage uses, on
an mbarrier nothing arrives on; after a short limit it reports the time-out
bit and returns.  The context must stay usable: a normal call afterwards is
checked against the oracle."""
import time

import pytest
import torch

from linear_diffusion_cross_b200 import binding as B

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("limit_ns", [1_000_000, 20_000_000])
def test_bounded_wait_times_out_and_reports(limit_ns):
    status = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    B.fldce_selftest_wait(limit_ns, status)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(status) == 1
    assert dt >= limit_ns / 1e9 * 0.9
    assert dt < 5.0


def test_context_usable_after_timeout():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.fldce_selftest_wait(1_000_000, status)
    from tests.test_parity_gpu import _full_compare, _small
    from tests._parity import run_gpu
    wl = _small(200, 64, 500, seed=11)
    g = run_gpu(wl)
    _full_compare(wl, g, "bf16")
    assert int(status) == 1
