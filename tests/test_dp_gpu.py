"""The data-parallel step through the library on one GPU (a one-rank NCCL
group): the job-wide count, the dW-ready event with dW computed before dH,
and the side-stream reduction, against the oracle and the plain call."""
import socket

import pytest
import torch
import torch.distributed as dist

import oracle.fldce_oracle as O
from linear_diffusion_cross_b200 import binding as B
from linear_diffusion_cross_b200 import synth
from linear_diffusion_cross_b200.dp import LibraryKernels, fwd_bwd_data_parallel
from tests._parity import GRAD_TOL, LOSS_RTOL, f64, maxabs_err

pytestmark = pytest.mark.gpu


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("chunk,use_bias,total", [(0, False, 0.0), (128, True, 0.0),
                                                  (100, True, 500.0)])
def test_dp_step_one_rank(chunk, use_bias, total):
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_port()}", rank=0,
                            world_size=1)
    try:
        r = synth.Recipe("dp", 1, 300, 128, 1003, torch.bfloat16, 0.1, 1e-3)
        wl = synth.make(r, 7, label_smoothing=0.1)
        b = (0.3 * torch.randn(wl.V, generator=torch.Generator().manual_seed(7))).bfloat16()
        plan = B.Plan(wl.D, wl.V, wl.N, chunk_N=chunk, label_smoothing=0.1, device=dev)
        args = (wl.H.to(dev), wl.W.to(dev), wl.target.to(dev), wl.p_mask.to(dev))
        bias = b.to(dev) if use_bias else None
        kern = LibraryKernels(plan)
        assert kern._event.cuda_event != 0
        out = fwd_bwd_data_parallel(kern, *args, total=total, bias=bias)
        torch.cuda.synchronize()
        ref = O.fldce(f64(wl.H), f64(wl.W), wl.target.numpy(), f64(wl.p_mask), total=total,
                      label_smoothing=0.1, bias=f64(b) if use_bias else None)
        assert abs(float(out["loss"][0]) - ref.loss) <= LOSS_RTOL * abs(ref.loss)
        assert maxabs_err(f64(out["dH"]), ref.dH) <= GRAD_TOL["bf16"]
        assert maxabs_err(f64(out["dW"]), ref.dW) <= GRAD_TOL["bf16"]
        if use_bias:
            assert maxabs_err(f64(out["db"]), ref.db) <= GRAD_TOL["bf16"]
        # dW computed before dH (event path) equals the plain call's result
        plain = plan.fwd_bwd(*args, total if total > 0 else 0.0, bias=bias)
        torch.cuda.synchronize()
        assert torch.equal(plain["dW"], out["dW"]) and torch.equal(plain["dH"], out["dH"])
    finally:
        dist.destroy_process_group()


def test_dw_ready_event_fires_after_dw_is_final():
    """The library records the event once dW is final: a copy of dW taken on
    another stream right after the event equals the dW the call returns, even
    while dH (computed after dW in this mode) is still running."""
    dev = torch.device("cuda", 0)
    r = synth.Recipe("ev", 1, 4096, 2048, 32000, torch.bfloat16, 0.02, 1e-3)
    wl = synth.make(r, 8)
    plan = B.Plan(wl.D, wl.V, wl.N, device=dev)
    ev = torch.cuda.Event()
    ev.record(torch.cuda.current_stream(dev))
    side = torch.cuda.Stream(device=dev)
    args = (wl.H.to(dev), wl.W.to(dev), wl.target.to(dev), wl.p_mask.to(dev))
    out = plan.outputs(wl.N)
    out["dW"].zero_()
    plan.fwd_bwd(*args, wl.total, out=out, dw_ready_event=ev)
    side.wait_event(ev)
    with torch.cuda.stream(side):
        snap = out["dW"].clone()
    torch.cuda.synchronize()
    assert torch.equal(snap, out["dW"]) and torch.count_nonzero(snap) > 0
    with pytest.raises(ValueError):
        B.make_call(dw_ready_event=torch.cuda.Event())
