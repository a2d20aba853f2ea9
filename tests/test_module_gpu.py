"""The PyTorch module / autograd front end on the GPU against the oracle:
loss, x.grad and weight.grad, upstream gradients, reductions, EOB weighting."""
import numpy as np
import pytest
import torch

import oracle.fldce_oracle as O
from linear_diffusion_cross_b200 import synth
from linear_diffusion_cross_b200.module import FusedLinearDiffusionCrossEntropyLoss
from tests._parity import GRAD_TOL, LOSS_RTOL, maxabs_err

pytestmark = pytest.mark.gpu


def _wl(seed=0, B=3, T=100, D=128, V=999, dtype=torch.bfloat16, **kw):
    r = synth.Recipe("module", B, T, D, V, dtype, 0.1, 1e-3)
    return synth.make(r, seed, **kw)


def _run(wl, module, scale=1.0, p_mask=True, eob=None, three_d=True):
    dev = torch.device("cuda")
    Bsz = 3
    x = wl.H.to(dev)
    y = wl.target.to(dev)
    p = wl.p_mask.to(dev) if p_mask else None
    if three_d:
        x = x.reshape(Bsz, -1, wl.D)
        y = y.reshape(Bsz, -1)
        p = None if p is None else p.reshape(Bsz, -1)
    x = x.clone().requires_grad_(True)
    W = wl.W.to(dev).clone().requires_grad_(True)
    kw = {} if eob is None else dict(eob_token_id=eob[0], eob_weight=eob[1])
    loss = module(x, y, W, p_mask=p, **kw)
    (loss * scale).backward()
    torch.cuda.synchronize()
    return loss.detach().cpu(), x.grad.reshape(-1, wl.D).cpu(), W.grad.cpu()


def _oracle(wl, module, scale=1.0, p_mask=True, eob=None):
    H, W = wl.H.double().numpy(), wl.W.double().numpy()
    y = wl.target.numpy()
    p = wl.p_mask.double().numpy() if p_mask else np.ones(wl.N)
    if eob is not None:
        p = p.copy()
        p[y == eob[0]] /= eob[1]
    total = 0.0 if module.reduction == "mean" else 1.0
    return O.fldce(H, W, y, p, total=total, logit_scale=module.logit_scale,
                   label_smoothing=module.label_smoothing, ignore_index=module.ignore_index,
                   grad_out=scale)


def _check(got, ref, key="bf16"):
    loss, dH, dW = got
    assert abs(float(loss) - ref.loss) <= LOSS_RTOL * abs(ref.loss)
    assert maxabs_err(dH.double().numpy(), ref.dH) <= GRAD_TOL[key]
    assert maxabs_err(dW.double().numpy(), ref.dW) <= GRAD_TOL[key]


@pytest.mark.parametrize("kw,scale", [
    (dict(), 1.0),
    (dict(label_smoothing=0.1, logit_scale=0.5), 1.0),
    (dict(), 2.5),
    (dict(reduction="sum"), 0.25),
])
def test_module_matches_oracle(kw, scale):
    wl = _wl(1)
    m = FusedLinearDiffusionCrossEntropyLoss(**kw)
    _check(_run(wl, m, scale), _oracle(wl, m, scale))


def test_module_default_p_mask_is_plain_ce():
    wl = _wl(2)
    m = FusedLinearDiffusionCrossEntropyLoss()
    _check(_run(wl, m, p_mask=False), _oracle(wl, m, p_mask=False))


def test_module_eob_weighting():
    wl = _wl(3)
    y = wl.target
    eob_tok = int(y[y != -100][0])
    y[torch.nonzero(y != -100).flatten()[1::5]] = eob_tok   # several EOB targets
    m = FusedLinearDiffusionCrossEntropyLoss(label_smoothing=0.05)
    eob = (eob_tok, 3.0)
    _check(_run(wl, m, eob=eob), _oracle(wl, m, eob=eob))
    _check(_run(wl, m, p_mask=False, eob=eob), _oracle(wl, m, p_mask=False, eob=eob))


def test_module_fp32():
    wl = _wl(4, T=20, D=64, V=300, dtype=torch.float32)
    m = FusedLinearDiffusionCrossEntropyLoss(label_smoothing=0.2)
    _check(_run(wl, m, 1.5), _oracle(wl, m, 1.5), key="fp32")


def test_module_bias():
    wl = _wl(6)
    g = torch.Generator().manual_seed(6)
    b = (0.5 * torch.randn(wl.V, generator=g)).to(torch.bfloat16)
    m = FusedLinearDiffusionCrossEntropyLoss(label_smoothing=0.1)
    dev = torch.device("cuda")
    x = wl.H.to(dev).requires_grad_(True)
    W = wl.W.to(dev).requires_grad_(True)
    bt = b.to(dev).requires_grad_(True)
    loss = m(x, wl.target.to(dev), W, bt, p_mask=wl.p_mask.to(dev))
    (loss * 2.0).backward()
    torch.cuda.synchronize()
    ref = O.fldce(wl.H.double().numpy(), wl.W.double().numpy(), wl.target.numpy(),
                  wl.p_mask.double().numpy(), total=0.0, label_smoothing=0.1, grad_out=2.0,
                  bias=b.double().numpy())
    assert abs(float(loss.detach()) - ref.loss) <= LOSS_RTOL * abs(ref.loss)
    assert maxabs_err(x.grad.double().cpu().numpy(), ref.dH) <= GRAD_TOL["bf16"]
    assert maxabs_err(W.grad.double().cpu().numpy(), ref.dW) <= GRAD_TOL["bf16"]
    assert maxabs_err(bt.grad.double().cpu().numpy(), ref.db) <= GRAD_TOL["bf16"]
    with torch.no_grad():
        l2 = m(x, wl.target.to(dev), W, bt, p_mask=wl.p_mask.to(dev))
    assert abs(float(l2) - ref.loss) <= LOSS_RTOL * abs(ref.loss)


def test_module_no_grad_runs_forward_only():
    wl = _wl(5)
    m = FusedLinearDiffusionCrossEntropyLoss()
    dev = torch.device("cuda")
    with torch.no_grad():
        loss = m(wl.H.to(dev), wl.target.to(dev), wl.W.to(dev), p_mask=wl.p_mask.to(dev))
    ref = _oracle(wl, m)
    assert abs(float(loss) - ref.loss) <= LOSS_RTOL * abs(ref.loss)
