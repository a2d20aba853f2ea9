"""Vocabulary-parallel loss on one GPU: two (uneven) vocabulary shards run
one after the other; their statistics are gathered by stacking them (what the
all-gather does across ranks); each shard's backward yields its dW and db
rows and a partial dH.  Summed / concatenated, everything must match the
oracle on the whole vocabulary, and the loss must be the same on both
shards."""
import numpy as np
import pytest
import torch

import oracle.fldce_oracle as O
from linear_diffusion_cross_b200 import binding as B
from linear_diffusion_cross_b200 import synth
from tests._parity import GRAD_TOL, LOSS_RTOL, ROW_TOL, f64, maxabs_err

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


@pytest.mark.parametrize("N,D,V,cut,chunk,dtype,eps", [
    (300, 136, 1003, 513, 0, torch.bfloat16, 0.1),
    (260, 64, 2049, 1024, 128, torch.bfloat16, 0.0),
    (70, 64, 257, 100, 0, torch.float32, 0.2),
])
def test_two_shards_match_whole_vocabulary(N, D, V, cut, chunk, dtype, eps):
    wl = synth.make(synth.Recipe("vp", 1, N, D, V, dtype, 0.1, 1e-3), N, label_smoothing=eps,
                    logit_scale=0.8, grad_out=1.2, total=0.0)
    b = (0.3 * torch.randn(V, generator=torch.Generator().manual_seed(N))).to(dtype)
    H, y, p = wl.H.to(DEV), wl.target.to(DEV), wl.p_mask.to(DEV)
    shards = [(0, cut), (cut, V)]
    plans, stats = [], []
    for a, e in shards:
        plan = B.Plan(D, e - a, N, dtype=dtype, chunk_N=chunk, logit_scale=0.8,
                      label_smoothing=eps, dh_fp32=True, vocab_start=a, vocab_total=V,
                      device=DEV)
        plans.append(plan)
        st = torch.empty(N, 8, device=DEV)
        call = B.make_call(H=H, W=wl.W[a:e].to(DEV), bias=b[a:e].to(DEV), target=y, p_mask=p,
                           N=N, workspace=plan.workspace, workspace_bytes=plan.workspace_bytes)
        B.fldce_vp_stats(plan.handle, call, st)
        stats.append(st)
    all_stats = torch.stack(stats)
    outs = []
    for (a, e), plan in zip(shards, plans):
        out = {"loss": torch.empty(1, device=DEV), "lse": torch.empty(N, device=DEV),
               "argmax": torch.empty(N, dtype=torch.int32, device=DEV),
               "loss_per_token": torch.empty(N, device=DEV),
               "dH": torch.empty(N, D, device=DEV),
               "dW": torch.empty(e - a, D, device=DEV, dtype=dtype),
               "db": torch.empty(e - a, device=DEV, dtype=dtype),
               "err": torch.empty(2, dtype=torch.int32, device=DEV)}
        call = B.make_call(H=H, W=wl.W[a:e].to(DEV), bias=b[a:e].to(DEV), target=y, p_mask=p,
                           N=N, total=0.0, grad_out=1.2, loss=out["loss"],
                           loss_per_token=out["loss_per_token"], lse=out["lse"],
                           argmax=out["argmax"], dH=out["dH"], dW=out["dW"], db=out["db"],
                           workspace=plan.workspace, workspace_bytes=plan.workspace_bytes,
                           err_count=out["err"])
        B.fldce_vp_fwd_bwd(plan.handle, call, all_stats, 2)
        outs.append(out)
    torch.cuda.synchronize()
    ref = O.fldce(f64(wl.H), f64(wl.W), wl.target.numpy(), f64(wl.p_mask), total=0.0,
                  logit_scale=0.8, label_smoothing=eps, grad_out=1.2, bias=f64(b))
    key = "bf16" if dtype == torch.bfloat16 else "fp32"
    for o in outs:
        assert abs(float(o["loss"][0]) - ref.loss) <= LOSS_RTOL * abs(ref.loss)
        assert maxabs_err(f64(o["lse"]), ref.lse) <= ROW_TOL[key]
        assert maxabs_err(f64(o["loss_per_token"]), ref.loss_per_token) <= ROW_TOL[key]
        clear = ref.top2_gap > 1e-3
        assert np.array_equal(o["argmax"].cpu().numpy()[clear], ref.argmax[clear])
    assert torch.equal(outs[0]["loss"], outs[1]["loss"])
    dH = f64(outs[0]["dH"]) + f64(outs[1]["dH"])
    assert maxabs_err(dH, ref.dH) <= GRAD_TOL[key]
    dW = np.concatenate([f64(o["dW"]) for o in outs])
    assert maxabs_err(dW, ref.dW) <= GRAD_TOL[key]
    db = np.concatenate([f64(o["db"]) for o in outs])
    assert maxabs_err(db, ref.db) <= GRAD_TOL[key]


def test_sharded_plan_rejects_plain_calls_and_bad_ranges():
    plan = B.Plan(64, 100, 16, vocab_start=100, vocab_total=300, device=DEV)
    out = plan.outputs(16)
    with pytest.raises(B.FldceError):
        plan.fwd_bwd(torch.zeros(16, 64, device=DEV).bfloat16(),
                     torch.zeros(100, 64, device=DEV).bfloat16(),
                     torch.zeros(16, dtype=torch.int64, device=DEV), None, 16.0, out=out)
    with pytest.raises(B.FldceError):
        B.fldce_create(B.FLDCE_BF16, 64, 100, 16, vocab_start=250, vocab_total=300)


def test_two_shards_headline_size():
    """The headline workload (N = 8192, D = 2560, V = 151936) split into two
    uneven vocabulary shards (the cut at 70000, not a multiple of the tile),
    run one after the other: the loss of both shards equals the oracle's
    full-batch loss, every token's lse matches, and the summed partial dH rows
    and each shard's dW rows match the oracle on samples."""
    wl = synth.make("headline", 0)
    N, D, V = wl.N, wl.D, wl.V
    cut = 70000
    H, y, p = wl.H.to(DEV), wl.target.to(DEV), wl.p_mask.to(DEV)
    shards = [(0, cut), (cut, V)]
    plans, stats, Ws = [], [], []
    for a, e in shards:
        plan = B.Plan(D, e - a, N, dh_fp32=True, vocab_start=a, vocab_total=V, device=DEV)
        plans.append(plan)
        Ws.append(wl.W[a:e].contiguous().to(DEV))
        st = torch.empty(N, 8, device=DEV)
        call = B.make_call(H=H, W=Ws[-1], target=y, p_mask=p, N=N, workspace=plan.workspace,
                           workspace_bytes=plan.workspace_bytes)
        B.fldce_vp_stats(plan.handle, call, st)
        stats.append(st)
    all_stats = torch.stack(stats)
    outs = []
    for (a, e), plan, Wd in zip(shards, plans, Ws):
        out = {"loss": torch.empty(1, device=DEV), "lse": torch.empty(N, device=DEV),
               "dH": torch.empty(N, D, device=DEV),
               "dW": torch.empty(e - a, D, device=DEV, dtype=torch.bfloat16),
               "err": torch.empty(2, dtype=torch.int32, device=DEV)}
        call = B.make_call(H=H, W=Wd, target=y, p_mask=p, N=N, total=wl.total, grad_out=1.0,
                           loss=out["loss"], lse=out["lse"], dH=out["dH"], dW=out["dW"],
                           workspace=plan.workspace, workspace_bytes=plan.workspace_bytes,
                           err_count=out["err"])
        B.fldce_vp_fwd_bwd(plan.handle, call, all_stats, 2)
        torch.cuda.synchronize()
        outs.append({k: v.cpu() for k, v in out.items()})
        plan.close()
    Hf, Wf, yn, pf = f64(wl.H), f64(wl.W), wl.target.numpy(), f64(wl.p_mask)
    vr = synth.sample_rows(V, 64, 7, [0, cut - 1, cut, V - 1]).numpy()
    dWr, lse_all, lt_all = O.fldce_dw_rows(Hf, Wf, yn, pf, vr, total=wl.total)
    ref_loss = float(lt_all.sum())
    for o in outs:
        assert abs(float(o["loss"][0]) - ref_loss) <= LOSS_RTOL * abs(ref_loss)
        assert np.abs(f64(o["lse"]) - lse_all).max() <= ROW_TOL["bf16"] * np.abs(lse_all).max()
        assert o["err"].tolist() == [0, 0]
    dW = np.concatenate([f64(o["dW"]) for o in outs])
    assert maxabs_err(dW[vr], dWr) <= GRAD_TOL["bf16"]
    rows = synth.sample_rows(N, 96, 8, [0, N - 1]).numpy()
    ref = O.fldce_rows(Hf, Wf, yn, pf, rows, total=wl.total)
    dH = f64(outs[0]["dH"])[rows] + f64(outs[1]["dH"])[rows]
    assert maxabs_err(dH, ref.dH) <= GRAD_TOL["bf16"]
    ign = yn[rows] == wl.ignore_index
    assert np.all(dH[ign] == 0.0)
