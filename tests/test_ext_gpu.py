"""The extended call on the GPU against the oracle: the page's bias (and db),
a caller-supplied normaliser count (data-parallel use), the valid-token
count, the forward-only extended call, and in-place gradient scaling."""
import numpy as np
import pytest
import torch

import oracle.fldce_oracle as O
from linear_diffusion_cross_b200 import binding as B
from linear_diffusion_cross_b200 import synth
from tests._parity import GRAD_TOL, LOSS_RTOL, ROW_TOL, f64, maxabs_err

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def _wl(N, D, V, seed=0, dtype=torch.bfloat16, **kw):
    r = synth.Recipe("ext", 1, N, D, V, dtype, 0.1, 1e-3)
    return synth.make(r, seed, **kw)


def _bias(V, dtype, seed=0):
    g = torch.Generator().manual_seed(100 + seed)
    return (0.5 * torch.randn(V, generator=g)).to(dtype)


def _oracle(wl, bias=None, total=None):
    return O.fldce(f64(wl.H), f64(wl.W), wl.target.numpy(), f64(wl.p_mask),
                   total=wl.total if total is None else total, logit_scale=wl.logit_scale,
                   label_smoothing=wl.label_smoothing, ignore_index=wl.ignore_index,
                   grad_out=wl.grad_out, bias=None if bias is None else f64(bias))


@pytest.mark.parametrize("N,D,V,chunk,dw_fp32,dtype", [
    (300, 136, 1003, 0, False, torch.bfloat16),
    (300, 136, 1003, 128, False, torch.bfloat16),
    (260, 64, 2049, 100, True, torch.bfloat16),
    (70, 64, 257, 0, False, torch.float32),
    (70, 64, 257, 32, False, torch.float32),
])
def test_bias_and_db(N, D, V, chunk, dw_fp32, dtype):
    wl = _wl(N, D, V, seed=N, dtype=dtype, label_smoothing=0.1, logit_scale=0.7, grad_out=1.5)
    b = _bias(V, dtype, N)
    plan = B.Plan(D, V, N, dtype=dtype, chunk_N=chunk, logit_scale=wl.logit_scale,
                  label_smoothing=wl.label_smoothing, dw_fp32=dw_fp32, device=DEV)
    out = plan.fwd_bwd(wl.H.to(DEV), wl.W.to(DEV), wl.target.to(DEV), wl.p_mask.to(DEV),
                       wl.total, wl.grad_out, bias=b.to(DEV), want_argmax=True)
    torch.cuda.synchronize()
    ref = _oracle(wl, b)
    key = "bf16" if dtype == torch.bfloat16 else "fp32"
    assert abs(float(out["loss"][0]) - ref.loss) <= LOSS_RTOL * abs(ref.loss)
    assert maxabs_err(f64(out["dH"]), ref.dH) <= GRAD_TOL[key]
    assert maxabs_err(f64(out["dW"]), ref.dW) <= GRAD_TOL[key]
    assert maxabs_err(f64(out["db"]), ref.db) <= GRAD_TOL[key]
    assert maxabs_err(f64(out["lse"]), ref.lse) <= ROW_TOL[key]
    assert out["db"].dtype == (torch.float32 if dw_fp32 or dtype == torch.float32 else dtype)
    clear = ref.top2_gap > 1e-3
    assert np.array_equal(out["argmax"].cpu().numpy()[clear], ref.argmax[clear])


def test_bias_without_db_is_rejected():
    wl = _wl(64, 64, 300)
    plan = B.Plan(64, 300, 64, device=DEV)
    out = plan.outputs(64)
    call = B.make_call(H=wl.H.to(DEV), W=wl.W.to(DEV), bias=_bias(300, torch.bfloat16).to(DEV),
                       target=wl.target.to(DEV), N=64, total=64.0, grad_out=1.0,
                       loss=out["loss"], dH=out["dH"], dW=out["dW"], workspace=plan.workspace,
                       workspace_bytes=plan.workspace_bytes)
    with pytest.raises(B.FldceError) as e:
        B.fldce_fwd_bwd_ex(plan.handle, call)
    assert e.value.status == B.FLDCE_ERR_INVALID_ARG


def test_count_valid_and_supplied_count():
    wl = _wl(333, 64, 500, seed=3, total=0.0)
    plan = B.Plan(64, 500, 333, device=DEV)
    y = wl.target.to(DEV)
    cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    B.fldce_count_valid(plan.handle, y, wl.N, cnt)
    torch.cuda.synchronize()
    assert int(cnt) == wl.n_valid()
    # a caller-supplied count (here: as if three ranks held this many each)
    job = torch.tensor([3 * wl.n_valid()], dtype=torch.int32, device=DEV)
    out = plan.fwd_bwd(wl.H.to(DEV), wl.W.to(DEV), y, wl.p_mask.to(DEV), 0.0, count_dev=job)
    torch.cuda.synchronize()
    ref = _oracle(wl, total=float(3 * wl.n_valid()))
    assert abs(float(out["loss"][0]) - ref.loss) <= LOSS_RTOL * abs(ref.loss)
    assert maxabs_err(f64(out["dW"]), ref.dW) <= GRAD_TOL["bf16"]
    # an explicit total > 0 wins over the supplied count
    out2 = plan.fwd_bwd(wl.H.to(DEV), wl.W.to(DEV), y, wl.p_mask.to(DEV), 50.0, count_dev=job)
    torch.cuda.synchronize()
    ref2 = _oracle(wl, total=50.0)
    assert abs(float(out2["loss"][0]) - ref2.loss) <= LOSS_RTOL * abs(ref2.loss)


def test_forward_ex_with_bias():
    wl = _wl(200, 128, 700, seed=4, label_smoothing=0.2)
    b = _bias(700, torch.bfloat16, 4)
    plan = B.Plan(128, 700, 200, label_smoothing=0.2, device=DEV)
    loss = torch.empty(1, device=DEV)
    lse = torch.empty(200, device=DEV)
    call = B.make_call(H=wl.H.to(DEV), W=wl.W.to(DEV), bias=b.to(DEV), target=wl.target.to(DEV),
                       p_mask=wl.p_mask.to(DEV), N=200, total=wl.total, loss=loss, lse=lse,
                       workspace=plan.workspace, workspace_bytes=plan.workspace_bytes)
    B.fldce_forward_ex(plan.handle, call)
    torch.cuda.synchronize()
    ref = _oracle(wl, b)
    assert abs(float(loss) - ref.loss) <= LOSS_RTOL * abs(ref.loss)
    assert maxabs_err(f64(lse), ref.lse) <= ROW_TOL["bf16"]


@pytest.mark.parametrize("dtype,n", [(torch.bfloat16, 1000003), (torch.float32, 77), (torch.bfloat16, 5)])
def test_scale_in_place(dtype, n):
    x = torch.randn(n, device=DEV).to(dtype)
    x0 = x.clone()
    g = torch.tensor([2.5], device=DEV)
    B.fldce_scale(x, n, B.FLDCE_BF16 if dtype == torch.bfloat16 else B.FLDCE_FP32, g)
    torch.cuda.synchronize()
    assert torch.equal(x, (x0.float() * 2.5).to(dtype))
    one = torch.tensor([1.0], device=DEV)
    B.fldce_scale(x, n, B.FLDCE_BF16 if dtype == torch.bfloat16 else B.FLDCE_FP32, one)
    torch.cuda.synchronize()
    assert torch.equal(x, (x0.float() * 2.5).to(dtype))


# FLDCE_FLAG_DW_ACCUMULATE: two micro-batches with the same weight, dW and db
# accumulated over both, dH and the loss of the second call alone.
@pytest.mark.parametrize("D,V,chunk,dw_fp32,dtype,skip", [
    (136, 1003, 0, False, torch.bfloat16, False),     # one chunk: fp32 partial, then added
    (136, 1003, 128, False, torch.bfloat16, False),   # several chunks
    (64, 2049, 100, True, torch.bfloat16, False),     # fp32 dW takes the reduce-adds
    (64, 257, 32, False, torch.float32, False),       # CUDA-core path
    (136, 1003, 0, False, torch.bfloat16, True),      # compacted tokens
], ids=["bf16_1chunk", "bf16_chunks", "dw_fp32", "fp32", "skip"])
def test_dw_accumulate(D, V, chunk, dw_fp32, dtype, skip):
    w1 = _wl(300, D, V, seed=21, dtype=dtype, label_smoothing=0.1, grad_out=1.25)
    w2 = _wl(257, D, V, seed=22, dtype=dtype, label_smoothing=0.1, grad_out=1.25)
    w2.W = w1.W
    b = _bias(V, dtype, 3)
    plan = B.Plan(D, V, 300, dtype=dtype, chunk_N=chunk, label_smoothing=0.1, dw_fp32=dw_fp32,
                  skip_ignored=skip, dw_accumulate=True, device=DEV)
    out = plan.outputs(300)
    out["db"] = torch.zeros(V, device=DEV, dtype=torch.float32 if dw_fp32 else dtype)
    assert torch.count_nonzero(out["dW"]) == 0
    Wd, bd = w1.W.to(DEV), b.to(DEV)
    for wl in (w1, w2):
        o = {k: (v[:wl.N] if k in ("dH", "loss_per_token", "lse") else v) for k, v in out.items()}
        plan.fwd_bwd(wl.H.to(DEV), Wd, wl.target.to(DEV), wl.p_mask.to(DEV), wl.total,
                     wl.grad_out, out=o, bias=bd)
    torch.cuda.synchronize()
    r1, r2 = _oracle(w1, b), _oracle(w2, b)
    key = "bf16" if dtype == torch.bfloat16 else "fp32"
    assert maxabs_err(f64(out["dW"]), r1.dW + r2.dW) <= GRAD_TOL[key]
    assert maxabs_err(f64(out["db"]), r1.db + r2.db) <= GRAD_TOL[key]
    assert maxabs_err(f64(out["dH"][:w2.N]), r2.dH) <= GRAD_TOL[key]
    assert abs(float(out["loss"][0]) - r2.loss) <= LOSS_RTOL * abs(r2.loss)
    # a call with no tokens, and one whose tokens are all ignored, add nothing
    before = (out["dW"].clone(), out["db"].clone())
    empty = torch.empty(0, D, dtype=dtype, device=DEV)
    o0 = dict(out, dH=out["dH"][:0], loss_per_token=out["loss_per_token"][:0],
              lse=out["lse"][:0])
    plan.fwd_bwd(empty, Wd, torch.empty(0, dtype=torch.int64, device=DEV), None, 1.0,
                 out=o0, bias=bd)
    ign = torch.full((64,), -100, dtype=torch.int64, device=DEV)
    o1 = dict(out, dH=out["dH"][:64], loss_per_token=out["loss_per_token"][:64],
              lse=out["lse"][:64])
    plan.fwd_bwd(w1.H[:64].to(DEV), Wd, ign, None, 0.0, out=o1, bias=bd)
    torch.cuda.synchronize()
    assert torch.equal(out["dW"], before[0]) and torch.equal(out["db"], before[1])
