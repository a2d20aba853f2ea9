"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
on a synthetic workload and compare it with the float64 oracle.

Tolerances (written here, used by every parity test):
* loss: 1e-3 relative; per-token loss and lse: 1e-3 relative to max |ref|;
* dH, dW: max-abs-normalised error  max|gpu - ref| / max|ref|  <= 2e-2 for
  bf16 and <= 1e-5 for the fp32 element type;
* ignore masking: exact zeros; argmax: exact on every token whose float64
  top-2 logit gap exceeds ARGMAX_MARGIN (near-ties are reported, not compared).
"""
from __future__ import annotations

import numpy as np
import torch

from linear_diffusion_cross_b200 import binding as B
from linear_diffusion_cross_b200.synth import Workload

LOSS_RTOL = 1e-3
GRAD_TOL = {"bf16": 2e-2, "fp32": 1e-5}
ROW_TOL = {"bf16": 1e-3, "fp32": 1e-5}
ARGMAX_MARGIN = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def maxabs_err(got: np.ndarray, ref: np.ndarray) -> float:
    scale = float(np.abs(ref).max())
    if scale == 0.0:
        return float(np.abs(got).max())
    return float(np.abs(got - ref).max()) / scale


def run_gpu(wl: Workload, *, chunk_n=None, want_argmax=True, dw_fp32=False, p_mask_none=False,
            plan=None, max_N=None, dh_fp32=False):
    dev = torch.device("cuda")
    if plan is None:
        plan = B.Plan(wl.D, wl.V, max_N or max(wl.N, 1), dtype=wl.H.dtype,
                      chunk_N=wl.chunk_n if chunk_n is None else chunk_n,
                      logit_scale=wl.logit_scale, label_smoothing=wl.label_smoothing,
                      ignore_index=wl.ignore_index, dw_fp32=dw_fp32, dh_fp32=dh_fp32,
                      device=dev)
    H = wl.H.to(dev)
    W = wl.W.to(dev)
    y = wl.target.to(dev)
    p = None if p_mask_none else wl.p_mask.to(dev)
    out = plan.fwd_bwd(H, W, y, p, wl.total, wl.grad_out, want_argmax=want_argmax)
    torch.cuda.synchronize()
    res = {k: v.cpu() for k, v in out.items()}
    res["plan"] = plan
    return res


def oracle_inputs(wl: Workload, p_mask_none=False):
    p = np.ones(wl.N) if p_mask_none else f64(wl.p_mask)
    return f64(wl.H), f64(wl.W), wl.target.numpy(), p


def oracle_kw(wl: Workload):
    return dict(logit_scale=wl.logit_scale, label_smoothing=wl.label_smoothing,
                ignore_index=wl.ignore_index, grad_out=wl.grad_out)


def check_rows(wl: Workload, g: dict, ref, rows: np.ndarray, tol_key: str):
    """Per-token outputs of `rows` against the oracle (ref holds those rows)."""
    ign = wl.target.numpy()[rows] == wl.ignore_index
    lt = g["loss_per_token"].double().numpy()[rows]
    assert np.all(lt[ign] == 0.0), "ignored token with non-zero loss"
    dH = f64(g["dH"])[rows]
    assert np.all(dH[ign] == 0.0), "ignored token with non-zero dH row"
    e_lt = maxabs_err(lt, ref.loss_per_token)
    assert e_lt <= ROW_TOL[tol_key], f"loss_per_token err {e_lt}"
    e_lse = float(np.abs(g["lse"].double().numpy()[rows] - ref.lse).max() /
                  max(1.0, np.abs(ref.lse).max()))
    assert e_lse <= ROW_TOL[tol_key], f"lse err {e_lse}"
    e_dh = maxabs_err(dH, ref.dH)
    assert e_dh <= GRAD_TOL[tol_key], f"dH err {e_dh}"
    near = 0
    if "argmax" in g:
        am = g["argmax"].numpy()[rows].astype(np.int64)
        clear = ref.top2_gap > ARGMAX_MARGIN
        near = int((~clear).sum())
        bad = np.nonzero(clear & (am != ref.argmax))[0]
        assert bad.size == 0, f"argmax mismatch at rows {rows[bad][:8]}"
    return {"loss_per_token": e_lt, "lse": e_lse, "dH": e_dh, "argmax_near_ties": near}
