"""Properties that fix the GPU results without an oracle (they hold at any
size), and a canary for uninitialised workspace: the call must not depend on
what the workspace held before."""
import math

import numpy as np
import pytest
import torch

from linear_diffusion_cross_b200 import binding as B
from linear_diffusion_cross_b200 import synth
from tests._parity import GRAD_TOL, f64, maxabs_err, run_gpu

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def _wl(N, D, V, seed, **kw):
    return synth.make(synth.Recipe("inv", 1, N, D, V, torch.bfloat16, 0.1, 1e-3), seed, **kw)


def test_identical_weight_rows():
    """Every logit of a token is the same: lse = z + log V, CE = log V for
    any smoothing, and dH = sum_v G[n,v] W = 0 because the rows of G sum to 0."""
    wl = _wl(300, 256, 777, 21, label_smoothing=0.2, total=0.0)
    wl.W = wl.W[:1].expand(wl.V, wl.D).contiguous()
    g = run_gpu(wl)
    valid = (wl.target != wl.ignore_index).numpy()
    z = (f64(wl.H) @ f64(wl.W[0]))
    lse = g["lse"].double().numpy()
    assert np.abs(lse - (z + math.log(wl.V))).max() <= 1e-3 * max(1.0, np.abs(z).max())
    T = float(valid.sum())
    ce = g["loss_per_token"].double().numpy() * f64(wl.p_mask) * T
    assert np.abs(ce[valid] - math.log(wl.V)).max() <= 1e-3 * math.log(wl.V)
    # |dH| against the scale of one G-weighted row: G entries are O(1/(pT))
    scale = float(np.abs(f64(wl.W[0])).max() / (f64(wl.p_mask).min() * T))
    assert float(np.abs(f64(g["dH"])).max()) <= 2e-2 * scale


def test_vocabulary_permutation():
    """Permuting the rows of W together with the targets permutes the rows of
    dW and leaves the loss, lse and dH unchanged."""
    wl = _wl(400, 128, 1300, 22, label_smoothing=0.1)
    g1 = run_gpu(wl)
    perm = torch.randperm(wl.V, generator=torch.Generator().manual_seed(5))
    inv = torch.argsort(perm)
    wl2 = _wl(400, 128, 1300, 22, label_smoothing=0.1)
    wl2.W = wl.W[perm].contiguous()
    t = wl.target.clone()
    m = t != wl.ignore_index
    t[m] = inv[t[m]]
    wl2.target = t
    g2 = run_gpu(wl2)
    assert abs(float(g1["loss"][0]) - float(g2["loss"][0])) <= 1e-5 * abs(float(g1["loss"][0]))
    assert maxabs_err(f64(g2["lse"]), f64(g1["lse"])) <= 1e-5
    assert maxabs_err(f64(g2["dH"]), f64(g1["dH"])) <= GRAD_TOL["bf16"]
    assert maxabs_err(f64(g2["dW"]), f64(g1["dW"])[perm.numpy()]) <= GRAD_TOL["bf16"]


def test_token_permutation():
    """Permuting the tokens permutes dH and the per-token outputs and leaves
    dW and the loss unchanged (up to the order of the sums)."""
    wl = _wl(384, 128, 900, 23)
    g1 = run_gpu(wl)
    perm = torch.randperm(wl.N, generator=torch.Generator().manual_seed(6))
    wl2 = _wl(384, 128, 900, 23)
    wl2.H, wl2.target, wl2.p_mask = wl.H[perm], wl.target[perm], wl.p_mask[perm]
    g2 = run_gpu(wl2)
    assert abs(float(g1["loss"][0]) - float(g2["loss"][0])) <= 1e-5 * abs(float(g1["loss"][0]))
    torch.testing.assert_close(g2["loss_per_token"], g1["loss_per_token"][perm], rtol=1e-6,
                               atol=1e-7)
    torch.testing.assert_close(g2["lse"], g1["lse"][perm], rtol=1e-6, atol=1e-6)
    assert maxabs_err(f64(g2["dH"]), f64(g1["dH"])[perm.numpy()]) <= GRAD_TOL["bf16"]
    assert maxabs_err(f64(g2["dW"]), f64(g1["dW"])) <= GRAD_TOL["bf16"]


@pytest.mark.parametrize("opts", [
    dict(),                                          # one chunk
    dict(chunk_N=128),                               # several chunks, fp32 dW accumulator
    dict(chunk_N=128, dw_fp32=True, dh_fp32=True),
    dict(skip_ignored=True),
    dict(dw_accumulate=True),
    dict(dtype=torch.float32, chunk_N=96),
], ids=["one_chunk", "chunks", "fp32_out", "skip", "accumulate", "fp32"])
def test_workspace_garbage_does_not_leak(opts):
    """The same call on a workspace filled with NaN bit patterns and on one
    filled with zeros gives the same bits: nothing reads workspace it has
    not written first in this call."""
    opts = dict(opts)
    dtype = opts.pop("dtype", torch.bfloat16)
    r = synth.Recipe("canary", 1, 333, 128, 2100, dtype, 0.1, 1e-3)
    wl = synth.make(r, 24, label_smoothing=0.1)
    plan = B.Plan(wl.D, wl.V, wl.N, dtype=dtype, label_smoothing=0.1, device=DEV, **opts)
    H, W = wl.H.to(DEV), wl.W.to(DEV)
    y, p = wl.target.to(DEV), wl.p_mask.to(DEV)
    b = (0.3 * torch.randn(wl.V, generator=torch.Generator().manual_seed(7))).to(dtype).to(DEV)
    res = []
    for fill in (0xFF, 0x00):
        plan.workspace.fill_(fill)
        out = plan.outputs(wl.N, want_argmax=True)
        out["db"] = torch.zeros(wl.V, device=DEV,
                                dtype=torch.float32 if opts.get("dw_fp32") else dtype)
        plan.fwd_bwd(H, W, y, p, 0.0, 1.0, out=out, bias=b)
        torch.cuda.synchronize()
        res.append({k: v.clone() for k, v in out.items()})
    for k in res[0]:
        torch.testing.assert_close(res[0][k], res[1][k], rtol=0, atol=0, equal_nan=True, msg=k)
    assert torch.isfinite(res[0]["dW"].float()).all() and torch.isfinite(res[0]["dH"].float()).all()
