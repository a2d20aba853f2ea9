"""The fused call inside a CUDA graph: it allocates nothing and never
synchronises the host, so one step can be captured once and replayed.  The
replays must reproduce a direct call bit for bit (every reduction in the
library has a fixed order)."""
import pytest
import torch

from linear_diffusion_cross_b200 import binding as B
from linear_diffusion_cross_b200 import synth

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


@pytest.mark.parametrize("dtype,flags", [(torch.bfloat16, {}), (torch.bfloat16,
                                                                {"skip_ignored": True}),
                                         (torch.float32, {})],
                         ids=["bf16", "bf16_skip", "fp32"])
def test_captured_step_replays_bit_for_bit(dtype, flags):
    r = synth.Recipe("graph", 2, 300, 128, 1500, dtype, 0.1, 1e-3)
    wl = synth.make(r, 3, label_smoothing=0.1)
    plan = B.Plan(wl.D, wl.V, wl.N, dtype=dtype, chunk_N=128, label_smoothing=0.1, device=DEV,
                  **flags)
    H, W = wl.H.to(DEV), wl.W.to(DEV)
    y, p = wl.target.to(DEV), wl.p_mask.to(DEV)
    ref = plan.fwd_bwd(H, W, y, p, wl.total, 1.0)
    torch.cuda.synchronize()
    ref = {k: v.clone() for k, v in ref.items()}

    out = plan.outputs(wl.N)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):          # warm the host-side caches off the capture
        plan.fwd_bwd(H, W, y, p, wl.total, 1.0, out=out, stream=side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    for v in out.values():
        v.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        plan.fwd_bwd(H, W, y, p, wl.total, 1.0, out=out,
                     stream=torch.cuda.current_stream())
    for _ in range(2):
        for v in out.values():
            v.zero_()
        g.replay()
        torch.cuda.synchronize()
        for k in ("loss", "loss_per_token", "lse", "dH", "dW", "err"):
            # bit for bit; skipped tokens' lse is NaN on both sides
            torch.testing.assert_close(out[k], ref[k], rtol=0, atol=0, equal_nan=True,
                                       msg=k)
    del g
