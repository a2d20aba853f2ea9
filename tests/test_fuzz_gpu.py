"""Seeded random configurations against the float64 oracle: shapes with
ragged tiles in every dimension, and random combinations of the options
(label smoothing, negative and large logit scales, bias, p_mask or none,
explicit or counted normaliser, chunking -- including chunk starts off the
16-byte boundary of the per-token arrays --, fp32 dW / dH, compacted tokens,
the fused sweep 2 + dH kernel, the fp32 element type).  Each case is small
enough for the oracle to take a fraction of a second; the list is fixed by
its seeds."""
import numpy as np
import pytest
import torch

import oracle.fldce_oracle as O
from linear_diffusion_cross_b200 import binding as B
from linear_diffusion_cross_b200 import synth
from tests._parity import GRAD_TOL, LOSS_RTOL, ROW_TOL, f64, maxabs_err

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def _case(seed):
    rng = np.random.default_rng(1000 + seed)
    fp32 = seed % 7 == 6
    N = int(rng.integers(1, 700))
    D = int(8 * rng.integers(1, 65))
    V = int(rng.integers(1, 3000))
    opts = dict(
        label_smoothing=float(rng.choice([0.0, 0.0, 0.1, 1.0])),
        logit_scale=float(rng.choice([1.0, 1.0, -0.5, 2.5])),
        grad_out=float(rng.choice([1.0, 0.5, -2.0])),
        total=float(rng.choice([0.0, N, 1.0])),
    )
    chunk = int(rng.choice([0, 0, 64, 200]))
    bias = bool(rng.integers(0, 2))
    p_none = bool(rng.integers(0, 4) == 0)
    skip = (not fp32) and bool(rng.integers(0, 3) == 0)
    dw_fp32 = bool(rng.integers(0, 2))
    dh_fp32 = (not fp32) and (not skip) and bool(rng.integers(0, 3) == 0)
    fused = False
    if seed >= 28:
        # later seeds: chunk starts off the 16-byte boundary of the per-token
        # arrays, and the fused sweep 2 + dH kernel among the options
        chunk = int(rng.choice([0, 33, 99, 130]))
        fused = (not fp32) and (not skip) and bool(rng.integers(0, 2))
    return fp32, N, D, V, opts, chunk, bias, p_none, skip, dw_fp32, dh_fp32, fused


@pytest.mark.parametrize("seed", range(48))
def test_random_configuration(seed):
    fp32, N, D, V, opts, chunk, bias, p_none, skip, dw_fp32, dh_fp32, fused = _case(seed)
    dtype = torch.float32 if fp32 else torch.bfloat16
    r = synth.Recipe("fuzz", 1, N, D, V, dtype, 0.1, 1e-3)
    wl = synth.make(r, seed, **opts)
    b = (0.3 * torch.randn(V, generator=torch.Generator().manual_seed(seed))).to(dtype) \
        if bias else None
    plan = B.Plan(D, V, N, dtype=dtype, chunk_N=chunk, logit_scale=wl.logit_scale,
                  label_smoothing=wl.label_smoothing, dw_fp32=dw_fp32, dh_fp32=dh_fp32,
                  skip_ignored=skip, fused_dh=fused, device=DEV)
    p = None if p_none else wl.p_mask.to(DEV)
    out = plan.fwd_bwd(wl.H.to(DEV), wl.W.to(DEV), wl.target.to(DEV), p, wl.total,
                       wl.grad_out, bias=None if b is None else b.to(DEV), want_argmax=True)
    torch.cuda.synchronize()
    ref = O.fldce(f64(wl.H), f64(wl.W), wl.target.numpy(),
                  np.ones(N) if p_none else f64(wl.p_mask), total=wl.total,
                  logit_scale=wl.logit_scale, label_smoothing=wl.label_smoothing,
                  grad_out=wl.grad_out, bias=None if b is None else f64(b))
    key = "fp32" if fp32 else "bf16"
    ctx = (f"seed {seed}: N={N} D={D} V={V} {opts} chunk={chunk} bias={bias} "
           f"p_none={p_none} skip={skip} dw_fp32={dw_fp32} dh_fp32={dh_fp32} fused={fused}")
    loss = float(out["loss"][0])
    assert abs(loss - ref.loss) <= LOSS_RTOL * abs(ref.loss) + 1e-6, ctx
    assert maxabs_err(f64(out["dH"]), ref.dH) <= GRAD_TOL[key], ctx
    assert maxabs_err(f64(out["dW"]), ref.dW) <= GRAD_TOL[key], ctx
    if bias:
        assert maxabs_err(f64(out["db"]), ref.db) <= GRAD_TOL[key], ctx
    assert maxabs_err(f64(out["loss_per_token"]), ref.loss_per_token) <= ROW_TOL[key], ctx
    valid, _ = O.valid_tokens(wl.target.numpy(), V, wl.ignore_index)
    rows = valid if skip else np.ones(N, bool)
    lse = f64(out["lse"])[rows]
    assert np.abs(lse - ref.lse[rows]).max(initial=0.0) <= \
        ROW_TOL[key] * max(1.0, np.abs(ref.lse).max()), ctx
    am = out["argmax"].cpu().numpy()
    clear = rows & (ref.top2_gap > 1e-3)
    assert np.array_equal(am[clear], ref.argmax[clear]), ctx
    assert out["err"].tolist() == [ref.n_err, 0], ctx
    plan.close()
