"""GPU parity of the CUDA path (through the C ABI) against the float64 oracle,
on sizes the oracle finishes in seconds that still span several tiles and
ragged tails, plus the degenerate cases of the method."""
import numpy as np
import pytest
import torch

import oracle.fldce_oracle as O
from linear_diffusion_cross_b200 import binding as B
from linear_diffusion_cross_b200 import synth
from tests._parity import (ARGMAX_MARGIN, GRAD_TOL, LOSS_RTOL, ROW_TOL, check_rows, f64,
                           maxabs_err, oracle_inputs, oracle_kw, run_gpu)

pytestmark = pytest.mark.gpu


def _full_compare(wl, g, tol_key, p_mask_none=False):
    H, W, y, p = oracle_inputs(wl, p_mask_none)
    ref = O.fldce(H, W, y, p, total=wl.total, **oracle_kw(wl))
    loss = float(g["loss"][0])
    assert abs(loss - ref.loss) <= LOSS_RTOL * abs(ref.loss) + 1e-30, (loss, ref.loss)
    errs = check_rows(wl, g, ref, np.arange(wl.N), tol_key)
    dW = f64(g["dW"])
    errs["dW"] = maxabs_err(dW, ref.dW)
    assert errs["dW"] <= GRAD_TOL[tol_key], f"dW err {errs['dW']}"
    assert int(g["err"][0]) == ref.n_err and int(g["err"][1]) == 0
    errs["loss"] = abs(loss - ref.loss) / max(abs(ref.loss), 1e-30)
    return errs, ref


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tiny_fp32_config(seed):
    wl = synth.make("tiny", seed)
    g = run_gpu(wl)
    _full_compare(wl, g, "fp32")


def _small(N, D, V, seed=0, sigma=0.1, **kw):
    r = synth.Recipe("small", 1, N, D, V, torch.bfloat16, sigma, 1e-3)
    return synth.make(r, seed, **kw)


SMALL = [
    # N,   D,   V,    options
    (300, 136, 1003, {}),
    (256, 256, 1024, {"label_smoothing": 0.1, "logit_scale": 0.5, "total": 0.0}),
    (77, 64, 40, {"grad_out": 2.5}),
    (5, 8, 300, {"total": 1.0}),
    (513, 520, 2049, {"label_smoothing": 0.3, "logit_scale": 1.7, "grad_out": -0.75}),
    (1, 64, 1000, {}),
    (200, 64, 1000, {"logit_scale": -0.7, "label_smoothing": 0.1}),
    (50, 64, 1, {}),
    (96, 64, 500, {"label_smoothing": 1.0}),
]


def test_large_logits():
    """Logits in the hundreds (unit-scale W, logit_scale 30): the running
    maxima keep every exponential finite."""
    wl = _small(128, 64, 700, seed=13, sigma=1.0, logit_scale=30.0)
    g = run_gpu(wl)
    assert torch.isfinite(g["dH"].float()).all() and torch.isfinite(g["lse"]).all()
    _full_compare(wl, g, "bf16")


@pytest.mark.parametrize("N,D,V,kw", SMALL, ids=[f"N{a}_D{b}_V{c}" for a, b, c, _ in SMALL])
def test_small_bf16(N, D, V, kw):
    wl = _small(N, D, V, **kw)
    g = run_gpu(wl)
    _full_compare(wl, g, "bf16")


@pytest.mark.parametrize("chunk", [64, 128, 200, 0])
def test_chunk_invariance(chunk):
    wl = _small(300, 128, 777, seed=3, label_smoothing=0.05)
    g = run_gpu(wl, chunk_n=chunk)
    _full_compare(wl, g, "bf16")


@pytest.mark.parametrize("chunk", [100, 0])
def test_chunked_dw_fp32_output(chunk):
    wl = _small(260, 64, 500, seed=4)
    g = run_gpu(wl, chunk_n=chunk, dw_fp32=True)
    assert g["dW"].dtype == torch.float32
    _full_compare(wl, g, "bf16")


def test_p_mask_none_is_plain_ce():
    wl = _small(200, 64, 321, seed=5)
    g = run_gpu(wl, p_mask_none=True)
    _full_compare(wl, g, "bf16", p_mask_none=True)


def test_ignored_rows_never_read_p_mask():
    wl = _small(256, 64, 400, seed=6)
    ign = wl.target == wl.ignore_index
    p = wl.p_mask.clone()
    idx = torch.nonzero(ign).flatten()
    p[idx[0::2]] = float("nan")
    p[idx[1::2]] = 0.0
    wl.p_mask = p
    g = run_gpu(wl)
    assert torch.isfinite(g["dW"].float()).all() and torch.isfinite(g["dH"].float()).all()
    _full_compare(wl, g, "bf16")


def test_out_of_range_targets_counted_and_ignored():
    wl = _small(200, 64, 300, seed=7, total=0.0)
    t = wl.target.clone()
    valid = torch.nonzero(t != wl.ignore_index).flatten()
    t[valid[0]] = wl.V
    t[valid[1]] = -5
    t[valid[2]] = 10 ** 12
    wl.target = t
    g = run_gpu(wl)
    assert int(g["err"][0]) == 3
    assert float(g["loss_per_token"][valid[0]]) == 0.0
    _full_compare(wl, g, "bf16")


def test_all_ignored():
    wl = _small(130, 64, 300, seed=8)
    wl.target[:] = wl.ignore_index
    for total in (0.0, 7.0):
        wl.total = total
        g = run_gpu(wl)
        assert float(g["loss"][0]) == 0.0
        assert torch.count_nonzero(g["dH"]) == 0 and torch.count_nonzero(g["dW"]) == 0


def test_zero_tokens():
    plan = B.Plan(64, 300, 16)
    dev = torch.device("cuda")
    H = torch.empty(0, 64, dtype=torch.bfloat16, device=dev)
    W = torch.randn(300, 64, device=dev).bfloat16()
    y = torch.empty(0, dtype=torch.int64, device=dev)
    out = plan.outputs(0)
    out["dW"].fill_(1.0)
    plan.fwd_bwd(H, W, y, None, 0.0, out=out)
    torch.cuda.synchronize()
    assert float(out["loss"][0]) == 0.0
    assert torch.count_nonzero(out["dW"]) == 0


def test_loss_is_deterministic():
    wl = _small(400, 128, 1500, seed=9)
    g1 = run_gpu(wl)
    g2 = run_gpu(wl, plan=g1["plan"])
    assert torch.equal(g1["loss"], g2["loss"])
    assert torch.equal(g1["loss_per_token"], g2["loss_per_token"])
    assert torch.equal(g1["dH"], g2["dH"])


def test_forward_only_matches_fwd_bwd():
    wl = _small(300, 136, 1003, seed=10, label_smoothing=0.2)
    g = run_gpu(wl)
    plan = g["plan"]
    dev = torch.device("cuda")
    f = plan.forward(wl.H.to(dev), wl.W.to(dev), wl.target.to(dev), wl.p_mask.to(dev),
                     wl.total, want_argmax=True)
    torch.cuda.synchronize()
    assert torch.equal(f["loss"].cpu(), g["loss"])
    assert torch.equal(f["lse"].cpu(), g["lse"])
    assert torch.equal(f["argmax"].cpu(), g["argmax"])
    assert torch.equal(f["loss_per_token"].cpu(), g["loss_per_token"])
    # and directly against the float64 oracle
    H, W, y, p = oracle_inputs(wl)
    ref = O.fldce(H, W, y, p, total=wl.total, **oracle_kw(wl))
    fl = float(f["loss"][0])
    assert abs(fl - ref.loss) <= LOSS_RTOL * abs(ref.loss)
    assert maxabs_err(f["loss_per_token"].double().cpu().numpy(), ref.loss_per_token) <= \
        ROW_TOL["bf16"]
    assert float(np.abs(f["lse"].double().cpu().numpy() - ref.lse).max()) <= \
        ROW_TOL["bf16"] * max(1.0, float(np.abs(ref.lse).max()))
    clear = ref.top2_gap > ARGMAX_MARGIN
    assert np.array_equal(f["argmax"].cpu().numpy()[clear], ref.argmax[clear])
    ign = y == wl.ignore_index
    assert np.all(f["loss_per_token"].cpu().numpy()[ign] == 0.0)


def test_error_codes_leave_outputs_untouched():
    plan = B.Plan(64, 300, 16)
    dev = torch.device("cuda")
    H = torch.randn(32, 64, device=dev).bfloat16()
    W = torch.randn(300, 64, device=dev).bfloat16()
    y = torch.zeros(32, dtype=torch.int64, device=dev)
    out = plan.outputs(32)
    with pytest.raises(B.FldceError) as e:          # N > max_N
        plan.fwd_bwd(H, W, y, None, 0.0, out=out)
    assert e.value.status == B.FLDCE_ERR_INVALID_ARG
    with pytest.raises(B.FldceError) as e:          # workspace too small
        B.fldce_fwd_bwd(plan.handle, H[:16], W, y[:16], None, 16, 0.0, 1.0, out["loss"], None,
                        None, None, out["dH"], out["dW"], plan.workspace, 1024, None)
    assert e.value.status == B.FLDCE_ERR_WORKSPACE
    with pytest.raises(B.FldceError) as e:          # misaligned dH
        B.fldce_fwd_bwd(plan.handle, H[:16], W, y[:16], None, 16, 0.0, 1.0, out["loss"], None,
                        None, None, out["dH"].data_ptr() + 2, out["dW"], plan.workspace,
                        plan.workspace_bytes, None)
    assert e.value.status == B.FLDCE_ERR_ALIGN


def test_ignore_index_inside_vocabulary():
    """ignore_index may be a real vocabulary id (here 0): those targets carry
    no loss, and nothing else changes."""
    wl = _small(300, 64, 500, seed=12)
    t = wl.target.clone()
    t[t == -100] = 0
    t[3::7] = 0
    wl.target = t
    wl.ignore_index = 0
    g = run_gpu(wl)
    _full_compare(wl, g, "bf16")


# dH's vocabulary reduction is split into k ranges when that fills the last
# round of CTA pairs better: with 2 token tiles x 1 column tile, V = 3500 (55
# K steps) takes 3 splits and V = 5003 (79 K steps) takes 4.  Each split's
# fp32 partial is summed in split order, so dH is also bit-reproducible.
@pytest.mark.parametrize("V", [3500, 5003])
@pytest.mark.parametrize("dh_fp32", [False, True])
def test_split_dh(V, dh_fp32):
    wl = _small(300, 136, V, seed=14, label_smoothing=0.05)
    g = run_gpu(wl, dh_fp32=dh_fp32)
    assert g["dH"].dtype == (torch.float32 if dh_fp32 else torch.bfloat16)
    _full_compare(wl, g, "bf16")
    g2 = run_gpu(wl, plan=g["plan"])
    assert torch.equal(g["dH"], g2["dH"])


# With D = 4096 each 256-token tile of H is 2 MB; 22 token tiles (5500 tokens,
# the last tile ragged) exceed the sweeps' L2 block, so the sweeps walk the
# vocabulary under two blocks of 11 token tiles.  Every tile is still visited
# exactly once.
def test_sweeps_walk_token_tiles_in_l2_blocks():
    wl = _small(5500, 4096, 1500, seed=15, label_smoothing=0.1)
    g = run_gpu(wl)
    _full_compare(wl, g, "bf16")


# dH runs on 256 x 512 tiles (two MMAs per staged tile, one 512-column
# accumulator) when the schedule model prefers them over 256-wide ones: many
# tiles per pair and D a multiple of 512, or close to one.  These shapes take
# them: unsplit, in two vocabulary splits (bf16 and fp32 dH), and with D =
# 1000, whose last tile runs 24 columns past D.
@pytest.mark.parametrize("N,D,V,dh_fp32", [(4608, 2048, 1000, False), (2304, 2048, 5000, False),
                                           (2304, 2048, 5000, True), (9472, 1000, 1000, False)])
def test_wide_dh_tiles(N, D, V, dh_fp32):
    wl = _small(N, D, V, seed=16, label_smoothing=0.1, grad_out=0.5)
    g = run_gpu(wl, dh_fp32=dh_fp32)
    _full_compare(wl, g, "bf16")
