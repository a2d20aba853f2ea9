"""HostPipeline: inputs copied from pinned host memory on a copy stream while
the previous step computes.  Each step's loss must equal a plain call's on the
same inputs (same kernels, so bit for bit), for steps with different inputs."""
import pytest
import torch

from linear_diffusion_cross_b200 import binding as B
from linear_diffusion_cross_b200 import synth
from linear_diffusion_cross_b200.hostpipe import HostPipeline

pytestmark = pytest.mark.gpu


def test_pipelined_steps_match_plain_calls():
    dev = torch.device("cuda")
    r = synth.Recipe("pipe", 2, 1024, 512, 20000, torch.bfloat16, 0.05, 1e-3)
    wls = [synth.make(r, s) for s in range(5)]
    plan = B.Plan(512, 20000, 2048, device=dev)
    batches = [{"H": w.H.pin_memory(), "W": w.W.pin_memory(), "y": w.target.pin_memory(),
                "p": w.p_mask.pin_memory()} for w in wls]
    pipe = HostPipeline(plan, 2048)
    losses = pipe.run(batches, 2048.0)
    torch.cuda.synchronize()
    last_dW = pipe.out["dW"].clone()
    for w, got in zip(wls, losses.tolist()):
        ref = plan.fwd_bwd(w.H.to(dev), w.W.to(dev), w.target.to(dev), w.p_mask.to(dev), 2048.0)
        torch.cuda.synchronize()
        assert got == float(ref["loss"][0])
    assert torch.equal(last_dW, ref["dW"])
