"""fldce_fwd_bwd_noalloc: the entry point for callers that cannot allocate
device memory (a plugin whose host owns all device memory, a caller under a
budget that forbids allocations outside its pool, a binding that can only
pass the buffers it has).  Its scratch is a static device array inside the
library, so it takes no workspace.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test.  It passes on its own in a fresh
process and after the rest of the suite.
"""
import pytest
import torch

import oracle.fldce_oracle as O
from linear_diffusion_cross_b200 import binding as B
from linear_diffusion_cross_b200 import synth
from tests._parity import GRAD_TOL, LOSS_RTOL, ROW_TOL, maxabs_err

pytestmark = pytest.mark.gpu


def _workload(seed, N=300, D=136, V=1003):
    r = synth.Recipe("noalloc", 1, N, D, V, torch.bfloat16, 0.1, 1e-3)
    return synth.make(r, seed, label_smoothing=0.1)


def _outputs(plan, N):
    return plan.outputs(N, want_argmax=True)


def _compare(a, b):
    la, lb = float(a["loss"][0]), float(b["loss"][0])
    assert abs(la - lb) <= LOSS_RTOL * abs(lb)
    for k in ("dH", "dW"):
        e = maxabs_err(a[k].double().cpu().numpy(), b[k].double().cpu().numpy())
        assert e <= GRAD_TOL["bf16"], (k, e)
    for k in ("loss_per_token", "lse"):
        e = maxabs_err(a[k].double().cpu().numpy(), b[k].double().cpu().numpy())
        assert e <= ROW_TOL["bf16"], (k, e)
    assert torch.equal(a["argmax"], b["argmax"])
    assert a["err"].tolist() == [0, 0]


def test_noalloc_matches_workspace_entry_two_calls_in_a_row():
    dev = torch.device("cuda")
    # two different problems back to back through the static scratch, each
    # checked against the workspace entry point on the same inputs
    wls = [_workload(0), _workload(1, N=257, D=64, V=2050)]
    plans = []
    for wl in wls:
        plan = B.Plan(wl.D, wl.V, wl.N, label_smoothing=wl.label_smoothing, chunk_N=128,
                      device=dev)
        assert B.fldce_workspace_size(plan.handle, wl.N) <= B.FLDCE_STATIC_SCRATCH_BYTES
        plans.append(plan)
    results = []
    for wl, plan in zip(wls, plans):
        H, W = wl.H.to(dev), wl.W.to(dev)
        y, p = wl.target.to(dev), wl.p_mask.to(dev)
        ref = plan.fwd_bwd(H, W, y, p, wl.total, 1.5, want_argmax=True)
        got = _outputs(plan, wl.N)
        for k in ("dH", "dW"):
            got[k].fill_(float("nan"))
        B.fldce_fwd_bwd_noalloc(plan.handle, H, W, y, p, wl.N, wl.total, 1.5, got["loss"],
                                got["loss_per_token"], got["lse"], got["argmax"], got["dH"],
                                got["dW"], got["err"])
        torch.cuda.synchronize()
        results.append((got, ref))
    for got, ref in results:
        _compare(got, ref)
    # and each call directly against the float64 oracle
    for wl, (got, _) in zip(wls, results):
        o = O.fldce(wl.H.double().numpy(), wl.W.double().numpy(), wl.target.numpy(),
                    wl.p_mask.double().numpy(), total=wl.total, grad_out=1.5,
                    label_smoothing=wl.label_smoothing)
        assert abs(float(got["loss"][0]) - o.loss) <= LOSS_RTOL * abs(o.loss)
        for k, want in (("dH", o.dH), ("dW", o.dW)):
            e = maxabs_err(got[k].double().cpu().numpy(), want)
            assert e <= GRAD_TOL["bf16"], (k, e)
        e = maxabs_err(got["loss_per_token"].double().cpu().numpy(), o.loss_per_token)
        assert e <= ROW_TOL["bf16"], e


def test_noalloc_rejects_problems_beyond_the_static_scratch():
    plan = B.Plan(2560, 151936, 8192)           # one 8192-token chunk: a 2.5 GB G buffer
    assert B.fldce_workspace_size(plan.handle, 8192) > B.FLDCE_STATIC_SCRATCH_BYTES
    dev = torch.device("cuda")
    out = {"loss": torch.zeros(1, device=dev), "err": torch.zeros(2, dtype=torch.int32,
                                                                  device=dev)}
    with pytest.raises(B.FldceError) as e:
        B.fldce_fwd_bwd_noalloc(plan.handle, None, None, None, None, 8192, 0.0, 1.0, out["loss"],
                                None, None, None, None, None, out["err"])
    assert e.value.status == B.FLDCE_ERR_TOO_LARGE
    assert "static" in str(e.value)
