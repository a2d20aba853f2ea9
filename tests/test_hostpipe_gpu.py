"""HostPipeline: inputs copied from pinned host memory on an upload stream while
the previous step computes, and each step's results (loss, dH, dW) copied back
to pinned host memory on a download stream while the next step computes.
Every step's results must equal a plain call's on the same inputs (same
kernels, so bit for bit), for steps with different inputs; one step is also
checked against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle.fldce_oracle as O
from linear_diffusion_cross_b200 import binding as B
from linear_diffusion_cross_b200 import synth
from linear_diffusion_cross_b200.hostpipe import HostPipeline
from tests._parity import GRAD_TOL, LOSS_RTOL, maxabs_err

pytestmark = pytest.mark.gpu


def _setup(n_steps=5):
    dev = torch.device("cuda")
    r = synth.Recipe("pipe", 2, 1024, 512, 20000, torch.bfloat16, 0.05, 1e-3)
    wls = [synth.make(r, s) for s in range(n_steps)]
    plan = B.Plan(512, 20000, 2048, device=dev)
    batches = [{"H": w.H.pin_memory(), "W": w.W.pin_memory(), "y": w.target.pin_memory(),
                "p": w.p_mask.pin_memory()} for w in wls]
    return dev, wls, plan, batches


def test_pipelined_steps_match_plain_calls():
    dev, wls, plan, batches = _setup()
    pipe = HostPipeline(plan, 2048)
    results = [pipe.host_results() for _ in wls]
    losses = pipe.run(batches, 2048.0, results=results)
    torch.cuda.synchronize()
    last_dW = pipe.out["dW"].clone()
    for w, got, res in zip(wls, losses.tolist(), results):
        ref = plan.fwd_bwd(w.H.to(dev), w.W.to(dev), w.target.to(dev), w.p_mask.to(dev), 2048.0)
        torch.cuda.synchronize()
        assert got == float(ref["loss"][0])
        assert float(res["loss"][0]) == got
        assert torch.equal(res["dH"], ref["dH"].cpu())
        assert torch.equal(res["dW"], ref["dW"].cpu())
    assert torch.equal(last_dW, ref["dW"])


def test_shared_result_buffers_hold_the_last_step():
    """Two host result sets alternating over the steps (what the e2e bench
    does): each ends with the results of the last step that used it."""
    dev, wls, plan, batches = _setup(4)
    pipe = HostPipeline(plan, 2048)
    sets = [pipe.host_results(), pipe.host_results()]
    pipe.run(batches, 2048.0, results=[sets[i % 2] for i in range(len(wls))])
    torch.cuda.synchronize()
    for k, w in ((0, wls[2]), (1, wls[3])):
        ref = plan.fwd_bwd(w.H.to(dev), w.W.to(dev), w.target.to(dev), w.p_mask.to(dev), 2048.0)
        torch.cuda.synchronize()
        assert torch.equal(sets[k]["dW"], ref["dW"].cpu())
        assert torch.equal(sets[k]["dH"], ref["dH"].cpu())


def test_pipelined_results_match_the_oracle():
    dev = torch.device("cuda")
    r = synth.Recipe("pipe_small", 2, 160, 256, 3001, torch.bfloat16, 0.05, 1e-3)
    wls = [synth.make(r, s, label_smoothing=0.1) for s in range(3)]
    plan = B.Plan(256, 3001, 320, label_smoothing=0.1, device=dev)
    batches = [{"H": w.H.pin_memory(), "W": w.W.pin_memory(), "y": w.target.pin_memory(),
                "p": w.p_mask.pin_memory()} for w in wls]
    pipe = HostPipeline(plan, 320)
    results = [pipe.host_results() for _ in wls]
    pipe.run(batches, 320.0, results=results)
    torch.cuda.synchronize()
    for w, res in zip(wls, results):
        ref = O.fldce(w.H.double().numpy(), w.W.double().numpy(), w.target.numpy(),
                      w.p_mask.double().numpy(), total=320.0, label_smoothing=0.1)
        assert abs(float(res["loss"][0]) - ref.loss) <= LOSS_RTOL * abs(ref.loss)
        assert maxabs_err(res["dH"].double().numpy(), ref.dH) <= GRAD_TOL["bf16"]
        assert maxabs_err(res["dW"].double().numpy(), ref.dW) <= GRAD_TOL["bf16"]
        ign = w.target.numpy() == w.ignore_index
        assert np.all(res["dH"].double().numpy()[ign] == 0.0)
