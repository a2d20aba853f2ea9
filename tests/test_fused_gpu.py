"""FLDCE_FLAG_FUSED_DH on the GPU against the float64 oracle: sweep 2 fused with
the dH GEMM (G formed in shared memory and fed from there to the dH
tensor-core MMAs, dH partials reduce-added in fp32).  Ragged shapes (rows,
vocabulary and D not multiples of the tiles, D not a multiple of the 128-wide
dH chunks), several token chunks, label smoothing, logit scale, bias, fp32 dH
and a vocabulary shard, then the headline shape on sampled rows."""
import numpy as np
import pytest
import torch

import oracle.fldce_oracle as O
from linear_diffusion_cross_b200 import binding as B
from linear_diffusion_cross_b200 import synth
from tests._parity import (GRAD_TOL, LOSS_RTOL, ROW_TOL, check_rows, f64, maxabs_err,
                           oracle_inputs, oracle_kw)

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def _wl(N, D, V, seed=0, **kw):
    r = synth.Recipe("fused", 1, N, D, V, torch.bfloat16, 0.1, 1e-3)
    return synth.make(r, seed, **kw)


def _run(wl, fused, chunk=0, bias=None, dh_fp32=False):
    plan = B.Plan(wl.D, wl.V, wl.N, chunk_N=chunk, logit_scale=wl.logit_scale,
                  label_smoothing=wl.label_smoothing, dh_fp32=dh_fp32, fused_dh=fused,
                  device=DEV)
    out = plan.fwd_bwd(wl.H.to(DEV), wl.W.to(DEV), wl.target.to(DEV), wl.p_mask.to(DEV),
                       wl.total, wl.grad_out, want_argmax=True,
                       bias=None if bias is None else bias.to(DEV))
    torch.cuda.synchronize()
    res = {k: v.cpu() for k, v in out.items()}
    plan.close()
    return res


@pytest.mark.parametrize("N,D,V,chunk,eps,s,use_bias,dh_fp32", [
    (300, 136, 1003, 0, 0.1, 1.0, False, False),    # D = 128 + 8: a nearly empty dH chunk
    (300, 136, 1003, 128, 0.0, 0.7, False, False),  # three token chunks
    (257, 64, 2050, 0, 0.2, 1.3, True, False),      # bias and db
    (513, 256, 777, 200, 0.0, 1.0, False, True),    # fp32 dH
    (64, 512, 4096, 0, 0.0, 1.0, False, False),     # a single token tile
])
def test_fused_matches_oracle(N, D, V, chunk, eps, s, use_bias, dh_fp32):
    wl = _wl(N, D, V, seed=N + D, label_smoothing=eps, logit_scale=s, grad_out=1.25)
    bias = None
    if use_bias:
        g = torch.Generator().manual_seed(7)
        bias = (0.5 * torch.randn(V, generator=g)).bfloat16()
    got = _run(wl, True, chunk, bias, dh_fp32)
    H, W, y, p = oracle_inputs(wl)
    ref = O.fldce(H, W, y, p, total=wl.total, bias=None if bias is None else f64(bias),
                  **oracle_kw(wl))
    assert abs(float(got["loss"][0]) - ref.loss) <= LOSS_RTOL * abs(ref.loss)
    assert maxabs_err(f64(got["dH"]), ref.dH) <= GRAD_TOL["bf16"]
    assert maxabs_err(f64(got["dW"]), ref.dW) <= GRAD_TOL["bf16"]
    assert maxabs_err(f64(got["lse"]), ref.lse) <= ROW_TOL["bf16"]
    ign = y == wl.ignore_index
    assert np.all(f64(got["dH"])[ign] == 0.0)
    if use_bias:
        assert maxabs_err(f64(got["db"]), ref.db) <= GRAD_TOL["bf16"]
    assert got["err"].tolist() == [0, 0]
    assert got["dH"].dtype == (torch.float32 if dh_fp32 else torch.bfloat16)


def test_fused_and_staged_agree():
    """Same inputs through both designs: the loss and dW bit-identical (the
    same G reaches the same dW GEMM), dH equal up to the summation order of
    its fp32 partials."""
    wl = _wl(1000, 384, 5000, seed=3, label_smoothing=0.05)
    a = _run(wl, True)
    b = _run(wl, False)
    assert torch.equal(a["loss"], b["loss"])
    assert torch.equal(a["dW"], b["dW"])
    assert torch.equal(a["lse"], b["lse"])
    assert maxabs_err(f64(a["dH"]), f64(b["dH"])) <= 1e-2


def test_fused_vocab_shard():
    """A vocabulary shard's backward through the fused kernel: the partial dH
    of two shards sums to the oracle's dH."""
    from linear_diffusion_cross_b200.dp import LibraryShardKernels
    wl = _wl(300, 128, 1500, seed=5, label_smoothing=0.1)
    cut = 700
    stats, parts = [], []
    plans = []
    for v0, v1 in ((0, cut), (cut, wl.V)):
        plan = B.Plan(wl.D, v1 - v0, wl.N, label_smoothing=0.1, vocab_start=v0,
                      vocab_total=wl.V, dh_fp32=True, fused_dh=True, device=DEV)
        plans.append((plan, v0, v1))
        k = LibraryShardKernels(plan)
        stats.append(k.vp_stats(wl.H.to(DEV), wl.W[v0:v1].contiguous().to(DEV),
                                wl.target.to(DEV), wl.p_mask.to(DEV), None))
    all_stats = torch.stack(stats)
    for plan, v0, v1 in plans:
        k = LibraryShardKernels(plan)
        parts.append(k.vp_fwd_bwd(wl.H.to(DEV), wl.W[v0:v1].contiguous().to(DEV),
                                  wl.target.to(DEV), wl.p_mask.to(DEV), wl.total, 1.0, None,
                                  all_stats, None))
    torch.cuda.synchronize()
    H, W, y, p = oracle_inputs(wl)
    ref = O.fldce(H, W, y, p, total=wl.total, **oracle_kw(wl))
    dH = sum(f64(o["dH"]) for o in parts)
    assert maxabs_err(dH, ref.dH) <= GRAD_TOL["bf16"]
    dW = np.concatenate([f64(o["dW"]) for o in parts])
    assert maxabs_err(dW, ref.dW) <= GRAD_TOL["bf16"]
    assert abs(float(parts[0]["loss"][0]) - ref.loss) <= LOSS_RTOL * abs(ref.loss)


def test_fused_headline_sampled_rows():
    """The headline shape (N = 8192, D = 2560, V = 151936) through the fused
    kernel: sampled dH rows and per-token outputs against the oracle."""
    wl = synth.make("headline", 0)
    got = _run(wl, True)
    H, W, y, p = oracle_inputs(wl)
    valid, _ = O.valid_tokens(y, wl.V, wl.ignore_index)
    T = O.resolve_total(wl.total, valid)
    rows = synth.sample_rows(wl.N, 96, 5, [0, wl.N - 1]).numpy()
    ref = O.fldce_rows(H, W, y, p, rows, total=T, **oracle_kw(wl))
    check_rows(wl, got, ref, rows, "bf16")
    ign = torch.from_numpy(~valid)
    assert torch.count_nonzero(got["dH"][ign]) == 0
