"""The per-token kernels move targets, p_mask and per-token outputs as 128-bit
vectors where they are 16-byte aligned, and fall back to scalar accesses
elsewhere.  These cases force the fallbacks against the float64 oracle:

* token chunks whose starts are 8 or 4 bytes off a 16-byte boundary
  (chunk_N = 99 and 130), so the merge's four-row groups of some chunks are
  misaligned;
* caller arrays that start off a 16-byte boundary (targets 8 bytes off,
  p_mask and the per-token outputs 4 or 12 bytes off), which also exercises
  the head and tail elements of the target-pair and loss-sum kernels;
* a row count that is not a multiple of four (the merge's last group);
and checks that arrays below their natural alignment are refused."""
import numpy as np
import pytest
import torch

import oracle.fldce_oracle as O
from linear_diffusion_cross_b200 import binding as B
from linear_diffusion_cross_b200 import synth
from tests._parity import GRAD_TOL, LOSS_RTOL, ROW_TOL, f64, maxabs_err

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def _wl(N, D, V, seed):
    r = synth.Recipe("vecio", 1, N, D, V, torch.bfloat16, 0.1, 1e-3)
    return synth.make(r, seed, label_smoothing=0.1, total=0.0)


def _offset(t: torch.Tensor, k: int) -> torch.Tensor:
    """A copy of t on the device that starts k elements into a fresh buffer."""
    buf = torch.zeros(t.numel() + k + 4, dtype=t.dtype, device=DEV)
    v = buf[k:k + t.numel()]
    v.copy_(t.to(DEV))
    return v


def _check(wl, got, ref):
    assert abs(float(got["loss"][0]) - ref.loss) <= LOSS_RTOL * abs(ref.loss)
    assert maxabs_err(f64(got["loss_per_token"]), ref.loss_per_token) <= ROW_TOL["bf16"]
    assert np.abs(f64(got["lse"]) - ref.lse).max() <= ROW_TOL["bf16"] * max(1.0, np.abs(ref.lse).max())
    assert maxabs_err(f64(got["dH"]), ref.dH) <= GRAD_TOL["bf16"]
    assert maxabs_err(f64(got["dW"]), ref.dW) <= GRAD_TOL["bf16"]
    clear = ref.top2_gap > 1e-3
    assert np.array_equal(got["argmax"].cpu().numpy()[clear], ref.argmax[clear])
    ign = wl.target.numpy() == wl.ignore_index
    assert np.all(f64(got["loss_per_token"])[ign] == 0.0)


def _oracle(wl):
    return O.fldce(f64(wl.H), f64(wl.W), wl.target.numpy(), f64(wl.p_mask), total=0.0,
                   label_smoothing=wl.label_smoothing)


@pytest.mark.parametrize("N,chunk", [(397, 99), (523, 130), (258, 0), (5, 0)])
def test_misaligned_chunks_and_arrays(N, chunk):
    wl = _wl(N, 72, 1500, seed=N)
    plan = B.Plan(wl.D, wl.V, N, chunk_N=chunk, label_smoothing=wl.label_smoothing,
                  device=DEV)
    out = plan.outputs(N, want_argmax=True)
    # caller arrays off the 16-byte boundary, each at its natural alignment
    y = _offset(wl.target, 1)                   # 8 bytes off
    p = _offset(wl.p_mask, 3)                   # 12 bytes off
    lt = _offset(torch.zeros(N), 1)             # 4 bytes off
    lse = _offset(torch.zeros(N), 2)            # 8 bytes off
    am = _offset(torch.zeros(N, dtype=torch.int32), 3)
    B.fldce_fwd_bwd(plan.handle, wl.H.to(DEV), wl.W.to(DEV), y, p, N, 0.0, 1.0, out["loss"],
                    lt, lse, am, out["dH"], out["dW"], plan.workspace, plan.workspace_bytes,
                    out["err"])
    torch.cuda.synchronize()
    got = {"loss": out["loss"].cpu(), "loss_per_token": lt.cpu(), "lse": lse.cpu(),
           "argmax": am.cpu(), "dH": out["dH"].cpu(), "dW": out["dW"].cpu()}
    _check(wl, got, _oracle(wl))
    assert out["err"].tolist() == [0, 0]
    # and the same problem through aligned buffers gives the same numbers
    ref = plan.fwd_bwd(wl.H.to(DEV), wl.W.to(DEV), wl.target.to(DEV), wl.p_mask.to(DEV), 0.0,
                       want_argmax=True)
    torch.cuda.synchronize()
    assert torch.equal(ref["lse"].cpu(), got["lse"])
    assert torch.equal(ref["argmax"].cpu(), got["argmax"])
    assert torch.allclose(ref["loss_per_token"].cpu(), got["loss_per_token"], rtol=0, atol=0)
    plan.close()


def test_forward_count_with_misaligned_targets():
    wl = _wl(301, 64, 777, seed=9)
    plan = B.Plan(wl.D, wl.V, wl.N, device=DEV)
    count = torch.zeros(1, dtype=torch.int32, device=DEV)
    for k in (0, 1):
        y = _offset(wl.target, k)
        B.fldce_count_valid(plan.handle, y, wl.N, count)
        torch.cuda.synchronize()
        assert int(count[0]) == wl.n_valid()
    plan.close()


def test_below_natural_alignment_is_refused():
    wl = _wl(64, 64, 300, seed=1)
    plan = B.Plan(wl.D, wl.V, wl.N, device=DEV)
    out = plan.outputs(wl.N)
    raw = torch.zeros(wl.N * 8 + 16, dtype=torch.uint8, device=DEV)
    cases = {
        "target": dict(target=raw.data_ptr() + 4),
        "p_mask": dict(p_mask=raw.data_ptr() + 2),
        "loss_per_token": dict(loss_per_token=raw.data_ptr() + 1),
    }
    for name, kw in cases.items():
        args = dict(target=wl.target.to(DEV), p_mask=wl.p_mask.to(DEV),
                    loss_per_token=out["loss_per_token"])
        args.update(kw)
        with pytest.raises(B.FldceError) as e:
            B.fldce_fwd_bwd(plan.handle, wl.H.to(DEV), wl.W.to(DEV), args["target"],
                            args["p_mask"], wl.N, 0.0, 1.0, out["loss"], args["loss_per_token"],
                            None, None, out["dH"], out["dW"], plan.workspace,
                            plan.workspace_bytes, out["err"])
        assert e.value.status == B.FLDCE_ERR_ALIGN, name
    plan.close()
