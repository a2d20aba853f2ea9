"""FLDCE_FLAG_SKIP_IGNORED on the GPU against the oracle: the tokens that
carry no loss are compacted away on the device, and every output but lse and
argmax of the skipped tokens is the same (those read NaN and -1)."""
import numpy as np
import pytest
import torch

import oracle.fldce_oracle as O
from linear_diffusion_cross_b200 import binding as B
from linear_diffusion_cross_b200 import synth
from tests._parity import GRAD_TOL, LOSS_RTOL, ROW_TOL, f64, maxabs_err

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def _plan(wl, chunk=0, dw_fp32=False):
    h, ws = B.fldce_create(B.FLDCE_BF16, wl.D, wl.V, max(wl.N, 1), chunk_N=chunk,
                           logit_scale=wl.logit_scale, label_smoothing=wl.label_smoothing,
                           flags=B.FLDCE_FLAG_SKIP_IGNORED |
                           (B.FLDCE_FLAG_DW_FP32 if dw_fp32 else 0))
    return h, torch.empty(ws, dtype=torch.uint8, device=DEV)


def _run(wl, chunk=0, dw_fp32=False, bias=None):
    h, ws = _plan(wl, chunk, dw_fp32)
    N, D, V = wl.N, wl.D, wl.V
    out = {"loss": torch.empty(1, device=DEV),
           "loss_per_token": torch.full((N,), 7.0, device=DEV),
           "lse": torch.empty(N, device=DEV),
           "argmax": torch.empty(N, dtype=torch.int32, device=DEV),
           "dH": torch.full((N, D), 3.0, device=DEV).bfloat16(),
           "dW": torch.full((V, D), 3.0, device=DEV,
                            dtype=torch.float32 if dw_fp32 else torch.bfloat16),
           "db": torch.empty(V, device=DEV, dtype=torch.float32 if dw_fp32 else torch.bfloat16),
           "err": torch.empty(2, dtype=torch.int32, device=DEV)}
    call = B.make_call(H=wl.H.to(DEV), W=wl.W.to(DEV), bias=None if bias is None else bias.to(DEV),
                       target=wl.target.to(DEV), p_mask=wl.p_mask.to(DEV), N=N, total=wl.total,
                       grad_out=wl.grad_out, loss=out["loss"],
                       loss_per_token=out["loss_per_token"], lse=out["lse"],
                       argmax=out["argmax"], dH=out["dH"], dW=out["dW"],
                       db=out["db"] if bias is not None else None, workspace=ws,
                       workspace_bytes=ws.numel(), err_count=out["err"])
    B.fldce_fwd_bwd_ex(h, call)
    torch.cuda.synchronize()
    B.fldce_destroy(h)
    return {k: v.cpu() for k, v in out.items()}


def _check(wl, g, bias=None):
    ref = O.fldce(f64(wl.H), f64(wl.W), wl.target.numpy(), f64(wl.p_mask), total=wl.total,
                  logit_scale=wl.logit_scale, label_smoothing=wl.label_smoothing,
                  grad_out=wl.grad_out, bias=None if bias is None else f64(bias))
    valid, _ = O.valid_tokens(wl.target.numpy(), wl.V, -100)
    assert abs(float(g["loss"][0]) - ref.loss) <= LOSS_RTOL * abs(ref.loss) + 1e-30
    lt = g["loss_per_token"].double().numpy()
    assert np.all(lt[~valid] == 0.0)
    assert maxabs_err(lt, ref.loss_per_token) <= ROW_TOL["bf16"]
    dH = f64(g["dH"])
    assert np.all(dH[~valid] == 0.0)
    assert maxabs_err(dH, ref.dH) <= GRAD_TOL["bf16"]
    assert maxabs_err(f64(g["dW"]), ref.dW) <= GRAD_TOL["bf16"]
    if bias is not None:
        assert maxabs_err(f64(g["db"]), ref.db) <= GRAD_TOL["bf16"]
    lse = g["lse"].double().numpy()
    assert np.all(np.isnan(lse[~valid]))
    assert maxabs_err(lse[valid], ref.lse[valid]) <= ROW_TOL["bf16"]
    am = g["argmax"].numpy()
    assert np.all(am[~valid] == -1)
    clear = valid & (ref.top2_gap > 1e-3)
    assert np.array_equal(am[clear], ref.argmax[clear])
    assert g["err"].tolist()[1] == 0


def _wl(N, D, V, seed, **kw):
    return synth.make(synth.Recipe("skip", 1, N, D, V, torch.bfloat16, 0.1, 1e-3), seed, **kw)


@pytest.mark.parametrize("N,D,V,chunk", [(300, 136, 1003, 0), (513, 64, 2049, 128),
                                         (600, 128, 777, 100), (77, 64, 40, 0),
                                         (300, 136, 5003, 0), (5500, 4096, 1500, 0),
                                         (4608, 2048, 1000, 0)])
def test_skip_matches_oracle(N, D, V, chunk):
    wl = _wl(N, D, V, N, label_smoothing=0.1, logit_scale=0.7, grad_out=1.3)
    _check(wl, _run(wl, chunk))


def test_skip_with_bias_and_fp32_dw_and_count_total():
    wl = _wl(400, 128, 1500, 5, total=0.0)
    b = (0.4 * torch.randn(1500, generator=torch.Generator().manual_seed(5))).bfloat16()
    _check(wl, _run(wl, 128, dw_fp32=True, bias=b), bias=b)
    _check(wl, _run(wl, 0, bias=b), bias=b)


@pytest.mark.parametrize("n_valid", [0, 1, 3])
def test_skip_almost_all_ignored(n_valid):
    wl = _wl(300, 64, 500, 9)
    t = torch.full_like(wl.target, -100)
    t[torch.arange(n_valid) * 97] = torch.arange(n_valid) * 13 + 1
    wl.target = t
    g = _run(wl, 128)
    if n_valid == 0:
        assert float(g["loss"][0]) == 0.0
        assert torch.count_nonzero(g["dW"]) == 0 and torch.count_nonzero(g["dH"]) == 0
        assert torch.isnan(g["lse"]).all() and (g["argmax"] == -1).all()
    else:
        _check(wl, g)


def test_skip_fp32_is_unsupported():
    with pytest.raises(B.FldceError) as e:
        B.fldce_create(B.FLDCE_FP32, 64, 100, 10, flags=B.FLDCE_FLAG_SKIP_IGNORED)
    assert e.value.status == B.FLDCE_ERR_UNSUPPORTED
