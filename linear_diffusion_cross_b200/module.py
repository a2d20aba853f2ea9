"""PyTorch front end over the C ABI: the page's FusedLinearDiffusionCrossEntropyLoss.

The interface follows the page "fused_linear_diffusion_cross_entropy.py":
``FusedLinearDiffusionCrossEntropyLoss(ignore_index, label_smoothing,
logit_scale, num_chunks, reduction)`` and its
``forward(x, target, weight, bias=None, p_mask=None, eob_token_id=None,
eob_weight=1.0)``, backed by ``FusedLinearCrossEntropyFunction``:

* the forward computes the loss and both gradients in one library call
  (``fldce_fwd_bwd``) and saves the gradients;
* the backward multiplies them by the upstream gradient with the library's
  ``fldce_scale`` (skipped on the device when it is 1);
* with autograd off (or no input needing a gradient) only the loss sweep
  runs (``fldce_forward``).

Differences from the page, by design: ``num_chunks`` is replaced by
``chunk_n`` (tokens per chunk; 0 lets the library size it so the gradient
buffer stays within 4 GiB); the 'mean' normaliser is counted on the device
(no host sync); the whole smoothed cross-entropy is divided by p_mask.
PyTorch here only flattens, allocates and passes pointers.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import binding as B


class _PlanCache:
    """One plan and workspace per (device, shape, options), grown on demand.

    Calls that share a plan share its workspace: issue them on one stream.
    """

    def __init__(self):
        self._plans = {}

    def get(self, device, dtype, D, V, N, *, label_smoothing, logit_scale, ignore_index,
            chunk_n) -> B.Plan:
        key = (device, dtype, D, V, float(label_smoothing), float(logit_scale),
               int(ignore_index), int(chunk_n))
        plan = self._plans.get(key)
        if plan is None or plan.max_N < N:
            if plan is not None:
                plan.close()
            plan = B.Plan(D, V, max(N, 1), dtype=dtype, chunk_N=chunk_n,
                          logit_scale=logit_scale, label_smoothing=label_smoothing,
                          ignore_index=ignore_index, device=device)
            self._plans[key] = plan
        return plan


_CACHE = _PlanCache()


def _dtype_code(dtype: torch.dtype) -> int:
    if dtype == torch.bfloat16:
        return B.FLDCE_BF16
    if dtype == torch.float32:
        return B.FLDCE_FP32
    raise TypeError(f"unsupported dtype {dtype}: use bfloat16 (tensor cores) or float32")


class FusedLinearCrossEntropyFunction(torch.autograd.Function):
    """Loss of ``x @ weight.T`` under the diffusion-weighted cross-entropy,
    with the gradients computed in the forward (as on the page)."""

    @staticmethod
    def forward(ctx, x, target, weight, bias, p_mask, total: float, opts: dict):
        N, D = x.shape
        V = weight.shape[0]
        plan = _CACHE.get(x.device, x.dtype, D, V, N, **opts)
        stream = torch.cuda.current_stream(x.device)
        loss = torch.empty((), dtype=torch.float32, device=x.device)
        dH = torch.empty_like(x)
        dW = torch.empty_like(weight)
        db = None if bias is None else torch.empty_like(bias)
        err = torch.empty(2, dtype=torch.int32, device=x.device)
        call = B.make_call(H=x, W=weight, bias=bias, target=target, p_mask=p_mask, N=N,
                           total=float(total), grad_out=1.0, loss=loss, dH=dH, dW=dW, db=db,
                           workspace=plan.workspace, workspace_bytes=plan.workspace_bytes,
                           err_count=err, stream=stream)
        B.fldce_fwd_bwd_ex(plan.handle, call)
        if db is None:
            ctx.save_for_backward(dH, dW)
        else:
            ctx.save_for_backward(dH, dW, db)
        return loss

    @staticmethod
    def backward(ctx, do):
        saved = ctx.saved_tensors
        g = do.detach().to(torch.float32).reshape(1).contiguous()
        stream = torch.cuda.current_stream(saved[0].device)
        for t in saved:
            B.fldce_scale(t, t.numel(), _dtype_code(t.dtype), g, stream)
        db = saved[2] if len(saved) == 3 else None
        return saved[0], None, saved[1], db, None, None, None


def fused_linear_cross_entropy_loss(x: torch.Tensor, target: torch.Tensor,
                                    weight: torch.Tensor, bias: Optional[torch.Tensor] = None,
                                    p_mask: Optional[torch.Tensor] = None,
                                    ignore_index: int = -100, label_smoothing: float = 0.0,
                                    logit_scale: float = 1.0, chunk_n: int = 0,
                                    reduction: str = "mean") -> torch.Tensor:
    """x [N, D], target [N] int64, weight [V, D], bias [V] or None, p_mask [N]
    fp32 or None -> loss."""
    if reduction not in ("mean", "sum"):
        raise ValueError(f"reduction: {reduction} is not supported")
    if x.dim() != 2 or weight.dim() != 2 or x.shape[1] != weight.shape[1]:
        raise ValueError(f"x {tuple(x.shape)} and weight {tuple(weight.shape)} do not match")
    if x.dtype != weight.dtype:
        raise TypeError("x and weight must have the same dtype")
    if target.shape[0] != x.shape[0] or (p_mask is not None and p_mask.shape[0] != x.shape[0]):
        raise ValueError(f"x={tuple(x.shape)}, target={tuple(target.shape)}, "
                         f"p_mask={None if p_mask is None else tuple(p_mask.shape)}")
    if not x.is_cuda:
        raise RuntimeError("the fused linear diffusion cross-entropy runs on CUDA tensors only")
    _dtype_code(x.dtype)
    x = x.contiguous()
    weight = weight.contiguous()
    target = target.contiguous().to(torch.int64)
    if p_mask is not None:
        p_mask = p_mask.contiguous().to(torch.float32)
    if bias is not None:
        if bias.shape != (weight.shape[0],) or bias.dtype != weight.dtype:
            raise ValueError(f"bias {tuple(bias.shape)} {bias.dtype} does not match weight")
        bias = bias.contiguous()
    total = 0.0 if reduction == "mean" else 1.0
    opts = dict(label_smoothing=label_smoothing, logit_scale=logit_scale,
                ignore_index=ignore_index, chunk_n=chunk_n)
    needs_grad = x.requires_grad or weight.requires_grad or (
        bias is not None and bias.requires_grad)
    if torch.is_grad_enabled() and needs_grad:
        return FusedLinearCrossEntropyFunction.apply(x, target, weight, bias, p_mask, total, opts)
    N, D = x.shape
    plan = _CACHE.get(x.device, x.dtype, D, weight.shape[0], N, **opts)
    loss = torch.empty((), dtype=torch.float32, device=x.device)
    call = B.make_call(H=x, W=weight, bias=bias, target=target, p_mask=p_mask, N=N,
                       total=float(total), loss=loss, workspace=plan.workspace,
                       workspace_bytes=plan.workspace_bytes,
                       stream=torch.cuda.current_stream(x.device))
    B.fldce_forward_ex(plan.handle, call)
    return loss


class FusedLinearDiffusionCrossEntropyLoss(torch.nn.Module):
    """Drop-in module with the page's constructor and forward signature."""

    def __init__(self, ignore_index: int = -100, label_smoothing: float = 0.0,
                 logit_scale: float = 1.0, chunk_n: int = 0, reduction: str = "mean"):
        super().__init__()
        if reduction not in ("mean", "sum"):
            raise ValueError(f"reduction: {reduction} is not supported")
        self.ignore_index = ignore_index
        self.label_smoothing = label_smoothing
        self.logit_scale = logit_scale
        self.chunk_n = chunk_n
        self.reduction = reduction

    def forward(self, x: torch.Tensor, target: torch.Tensor, weight: torch.Tensor,
                bias: Optional[torch.Tensor] = None, p_mask: Optional[torch.Tensor] = None,
                eob_token_id: Optional[int] = None, eob_weight: float = 1.0) -> torch.Tensor:
        """x [B, T, D] (or [N, D]), target [B, T], p_mask [B, T] or None (= 1)."""
        x2 = x.reshape(-1, x.shape[-1])
        t2 = target.reshape(-1)
        p2 = None if p_mask is None else p_mask.reshape(-1)
        if eob_token_id is not None and eob_weight != 1.0:
            # the page's EOB weighting: loss[n] * eob_weight for EOB targets,
            # done by dividing their p_mask (a caller-side edit of the input)
            if p2 is None:
                p2 = torch.ones(t2.shape[0], dtype=torch.float32, device=x.device)
            p2 = p2.to(torch.float32).clone()
            is_eob = t2 == eob_token_id
            p2[is_eob] = p2[is_eob] / eob_weight
        return fused_linear_cross_entropy_loss(
            x2, t2, weight, bias, p2, ignore_index=self.ignore_index,
            label_smoothing=self.label_smoothing, logit_scale=self.logit_scale,
            chunk_n=self.chunk_n, reduction=self.reduction)
