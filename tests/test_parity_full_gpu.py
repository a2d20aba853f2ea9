"""GPU parity at the full workload sizes, in the launch configuration bench.py
times (default chunking, argmax on).  The oracle computes what it can one
row at a time:

* every sampled token's lse, loss and dH row;
* for every workload, sampled vocabulary rows of dW, element by element:
  always the last row (V - 1, the ragged tail of a vocabulary that is not a
  multiple of the tile width), target rows of valid tokens, and for the
  large workload a set of the rows drawn x8;
* the scalar loss against the oracle's full-batch sum, and every token's
  lse and per-token loss (the dW rows need the whole batch's lse anyway).

Properties that hold at any size are checked everywhere as well:

* ignored tokens: loss and dH row exactly zero (every token, not a sample);
* loss == sum of loss_per_token;
* every row of G sums to zero, so the column sums of dW vanish
  (|sum_v dW[v, :]| small against sum_v |dW[v, :]|).
"""
import time

import numpy as np
import pytest
import torch

import oracle.fldce_oracle as O
from linear_diffusion_cross_b200 import synth
from tests._parity import (GRAD_TOL, LOSS_RTOL, ROW_TOL, check_rows, f64, maxabs_err,
                           oracle_inputs, oracle_kw, run_gpu)

pytestmark = pytest.mark.gpu

N_SAMPLE_ROWS = 192
N_SAMPLE_VOCAB = 128


def _global_checks(wl, g):
    ign = (wl.target == wl.ignore_index).numpy()
    lt = g["loss_per_token"].double().numpy()
    assert np.all(lt[ign] == 0.0)
    dH = g["dH"]
    assert torch.count_nonzero(dH[torch.from_numpy(ign)]) == 0
    loss = float(g["loss"][0])
    assert abs(loss - lt.sum()) <= 1e-5 * abs(lt.sum())
    assert int(g["err"][0]) == 0 and int(g["err"][1]) == 0
    dW = g["dW"].float()
    colsum = dW.double().sum(0).abs()
    colabs = dW.double().abs().sum(0)
    ratio = float((colsum / colabs.clamp_min(1e-30)).max())
    assert ratio < 2e-2, f"dW column sums not ~0: {ratio}"
    return ratio


def _rows(wl, seed):
    must = [0, wl.N - 1]
    return synth.sample_rows(wl.N, N_SAMPLE_ROWS, seed, must).numpy()


@pytest.mark.parametrize("name", ["mid", "headline", "ragged", "large"])
def test_full_size(name):
    t0 = time.time()
    wl = synth.make(name, 0)
    g = run_gpu(wl)
    H, W, y, p = oracle_inputs(wl)
    valid, _ = O.valid_tokens(y, wl.V, wl.ignore_index)
    T = O.resolve_total(wl.total, valid)
    info = {"gen_and_gpu_s": time.time() - t0}
    info["dW_colsum_ratio"] = _global_checks(wl, g)

    rows = _rows(wl, 1)
    t1 = time.time()
    ref = O.fldce_rows(H, W, y, p, rows, total=T, **oracle_kw(wl))
    info.update(check_rows(wl, g, ref, rows, "bf16"))
    info["oracle_rows_s"] = time.time() - t1

    must = [wl.V - 1, wl.V - 2] + [int(v) for v in y[valid][:8]]
    if wl.peaky_rows is not None:
        # rows drawn x8: the peaky logits of the large workload
        pk = wl.peaky_rows.numpy()
        must += [int(v) for v in pk[np.linspace(0, pk.size - 1, 16).astype(np.int64)]]
    vr = synth.sample_rows(wl.V, N_SAMPLE_VOCAB, 2, must).numpy()
    t2 = time.time()
    dWr, lse_all, lt_all = O.fldce_dw_rows(H, W, y, p, vr, total=T, **oracle_kw(wl))
    info["oracle_dw_s"] = time.time() - t2
    e_dw = maxabs_err(f64(g["dW"])[vr], dWr)
    info["dW"] = e_dw
    if wl.peaky_rows is not None:
        pk_set = np.isin(vr, wl.peaky_rows.numpy())
        info["dW_peaky_rows"] = int(pk_set.sum())
        info["dW_peaky_err"] = maxabs_err(f64(g["dW"])[vr[pk_set]], dWr[pk_set])
    assert e_dw <= GRAD_TOL["bf16"], f"dW err {e_dw}"
    # every token: lse and per-token loss against the oracle's whole batch
    e_lse = float(np.abs(g["lse"].double().numpy() - lse_all).max() /
                  max(1.0, np.abs(lse_all).max()))
    e_lt = maxabs_err(g["loss_per_token"].double().numpy(), lt_all)
    info["lse_all"] = e_lse
    info["loss_per_token_all"] = e_lt
    assert e_lse <= ROW_TOL["bf16"], f"lse err {e_lse}"
    assert e_lt <= ROW_TOL["bf16"], f"loss_per_token err {e_lt}"
    loss_ref = float(lt_all.sum())
    loss = float(g["loss"][0])
    info["loss"] = abs(loss - loss_ref) / abs(loss_ref)
    assert abs(loss - loss_ref) <= LOSS_RTOL * abs(loss_ref), (loss, loss_ref)

    if name in ("ragged", "large"):
        # the same batch with the ignored tokens compacted away on the device
        # (FLDCE_FLAG_SKIP_IGNORED; for large, across its four token chunks)
        # against the same oracle values
        del g
        skip = _run_skip(wl)
        ls = float(skip["loss"][0])
        info["skip_loss"] = abs(ls - loss_ref) / abs(loss_ref)
        assert abs(ls - loss_ref) <= LOSS_RTOL * abs(loss_ref), (ls, loss_ref)
        e = maxabs_err(f64(skip["dW"])[vr], dWr)
        info["skip_dW"] = e
        assert e <= GRAD_TOL["bf16"], f"skip dW err {e}"
        vrows = rows[valid[rows]]
        e = maxabs_err(f64(skip["dH"])[vrows], ref.dH[valid[rows]])
        info["skip_dH"] = e
        assert e <= GRAD_TOL["bf16"], f"skip dH err {e}"
        ign = torch.from_numpy(~valid)
        assert torch.count_nonzero(skip["dH"][ign]) == 0
        assert torch.isnan(skip["lse"][ign]).all()
        lt = skip["loss_per_token"].double().numpy()
        assert maxabs_err(lt, lt_all) <= ROW_TOL["bf16"]
    print(name, info)


def _run_skip(wl):
    from linear_diffusion_cross_b200 import binding as B
    dev = torch.device("cuda")
    plan = B.Plan(wl.D, wl.V, wl.N, chunk_N=wl.chunk_n, logit_scale=wl.logit_scale,
                  label_smoothing=wl.label_smoothing, ignore_index=wl.ignore_index,
                  skip_ignored=True, device=dev)
    out = plan.fwd_bwd(wl.H.to(dev), wl.W.to(dev), wl.target.to(dev), wl.p_mask.to(dev),
                       wl.total, wl.grad_out)
    torch.cuda.synchronize()
    res = {k: v.cpu() for k, v in out.items()}
    assert res["err"].tolist() == [0, 0]
    plan.close()
    return res


def test_full_size_headline_skip_ignored():
    """The headline workload with FLDCE_FLAG_SKIP_IGNORED: same loss, dH rows
    and dW rows as the oracle; lse NaN and dH zero for every skipped token."""
    from linear_diffusion_cross_b200 import binding as B
    wl = synth.make("headline", 0)
    dev = torch.device("cuda")
    plan = B.Plan(wl.D, wl.V, wl.N, skip_ignored=True, device=dev)
    g = plan.fwd_bwd(wl.H.to(dev), wl.W.to(dev), wl.target.to(dev), wl.p_mask.to(dev),
                     wl.total, want_argmax=True)
    torch.cuda.synchronize()
    g = {k: v.cpu() for k, v in g.items()}
    H, W, y, p = oracle_inputs(wl)
    valid, _ = O.valid_tokens(y, wl.V, wl.ignore_index)
    ign = ~valid
    assert torch.count_nonzero(g["dH"][torch.from_numpy(ign)]) == 0
    assert torch.isnan(g["lse"][torch.from_numpy(ign)]).all()
    assert (g["argmax"][torch.from_numpy(ign)] == -1).all()
    rows = np.nonzero(valid)[0][synth.sample_rows(int(valid.sum()), N_SAMPLE_ROWS, 3).numpy()]
    ref = O.fldce_rows(H, W, y, p, rows, total=wl.total, **oracle_kw(wl))
    assert maxabs_err(f64(g["dH"])[rows], ref.dH) <= GRAD_TOL["bf16"]
    assert maxabs_err(g["loss_per_token"].double().numpy()[rows], ref.loss_per_token) <= 1e-3
    vr = synth.sample_rows(wl.V, N_SAMPLE_VOCAB, 4, [wl.V - 1]).numpy()
    dWr, _, lt_all = O.fldce_dw_rows(H, W, y, p, vr, total=wl.total, **oracle_kw(wl))
    assert maxabs_err(f64(g["dW"])[vr], dWr) <= GRAD_TOL["bf16"]
    loss_ref = float(lt_all.sum())
    assert abs(float(g["loss"][0]) - loss_ref) <= LOSS_RTOL * abs(loss_ref)
