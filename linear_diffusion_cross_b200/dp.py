"""Data-parallel fwd+bwd over token shards (torch.distributed, NCCL on GPUs).

The page's sequence-parallel style (``LinearLossParallel``) shards the tokens
(x and target) across ranks and replicates the weight and bias.  The loss and
the weight gradients are sums over tokens, so the one exchange step is a sum
over ranks:

1. the normaliser: with ``total <= 0`` (the page's 'mean' over non-ignored
   targets) each rank counts its valid targets on the device
   (``fldce_count_valid``) and the counts are summed across ranks, so every
   rank divides by the job-wide count with no host round trip;
2. each rank runs the fused call on its own tokens with that count;
   its dH rows are final (they depend only on its tokens);
3. dW, db and the loss are summed across ranks.  The library records an
   event as soon as dW (and db) are final -- it computes the last chunk's dW
   before its dH for this -- so their reduction runs on a side stream while
   dH is still being computed.

Every rank issues the same collectives in the same order.  ``LibraryKernels``
binds the per-rank steps to libfldce; the steps are an argument so the
exchange logic can be exercised with another implementation (the CPU tests
run it on gloo ranks).
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist

from . import binding as B


class LibraryKernels:
    """The per-rank steps, on the GPU through the C ABI."""

    def __init__(self, plan: B.Plan):
        self.plan = plan
        self._side = torch.cuda.Stream(device=plan.device)
        # torch creates the CUDA event on its first record; the library records
        # it by handle, so create it now (a record on an idle stream is free)
        self._event = torch.cuda.Event()
        self._event.record(torch.cuda.current_stream(plan.device))
        if not self._event.cuda_event:
            raise RuntimeError("could not create the dW-ready CUDA event")

    def count_valid(self, target: torch.Tensor) -> torch.Tensor:
        count = torch.empty(1, dtype=torch.int32, device=self.plan.device)
        B.fldce_count_valid(self.plan.handle, target, target.shape[0], count)
        return count

    def fwd_bwd(self, H, W, target, p_mask, total, grad_out, count, bias, out):
        return self.plan.fwd_bwd(H, W, target, p_mask, total, grad_out, out=out, bias=bias,
                                 count_dev=count, dw_ready_event=self._event)

    def reduce_weight_grads(self, tensors, group):
        """Sum dW (and db) over ranks on a side stream once they are final."""
        side = self._side
        side.wait_event(self._event)
        with torch.cuda.stream(side):
            for t in tensors:
                dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
        torch.cuda.current_stream(self.plan.device).wait_stream(side)
        for t in tensors:
            t.record_stream(side)


def fwd_bwd_data_parallel(kernels, H, W, target, p_mask, *, total: float = 0.0,
                          grad_out: float = 1.0, bias=None, out: Optional[dict] = None,
                          group=None) -> dict:
    """One data-parallel step.  H, target, p_mask: this rank's tokens; W, bias:
    replicated.  ``total > 0`` must already be the job-wide normaliser.
    Returns this rank's outputs with dW, db and loss summed over ranks.
    A plan that accumulates dW is refused: each step's sum over ranks would
    add the earlier steps' gradients once per rank."""
    plan = getattr(kernels, "plan", None)
    if plan is not None and getattr(plan, "dw_accumulate", False):
        raise ValueError("fwd_bwd_data_parallel needs a plan that overwrites dW")
    count = None
    if total <= 0:
        count = kernels.count_valid(target)
        dist.all_reduce(count, op=dist.ReduceOp.SUM, group=group)
    out = kernels.fwd_bwd(H, W, target, p_mask, total, grad_out, count, bias, out)
    grads = [out["dW"]] + ([out["db"]] if bias is not None else [])
    kernels.reduce_weight_grads(grads, group)
    dist.all_reduce(out["loss"], op=dist.ReduceOp.SUM, group=group)
    return out


# ---------------------------------------------------------------- vocabulary parallel

class LibraryShardKernels:
    """The per-rank steps of the vocabulary-parallel loss, through the C ABI.

    ``plan`` must cover this rank's vocabulary shard (made with vocab_start /
    vocab_total) and all tokens of the batch."""

    def __init__(self, plan: B.Plan):
        self.plan = plan

    def vp_stats(self, H, W, target, p_mask, bias):
        stats = torch.empty(H.shape[0], 8, dtype=torch.float32, device=self.plan.device)
        call = B.make_call(H=H, W=W, bias=bias, target=target, p_mask=p_mask, N=H.shape[0],
                           workspace=self.plan.workspace,
                           workspace_bytes=self.plan.workspace_bytes)
        B.fldce_vp_stats(self.plan.handle, call, stats)
        return stats

    def vp_fwd_bwd(self, H, W, target, p_mask, total, grad_out, bias, all_stats, out):
        N = H.shape[0]
        if out is None:
            out = self.plan.outputs(N)
            if bias is not None:
                out["db"] = torch.empty_like(bias)
        call = B.make_call(H=H, W=W, bias=bias, target=target, p_mask=p_mask, N=N,
                           total=float(total), grad_out=float(grad_out), loss=out["loss"],
                           loss_per_token=out.get("loss_per_token"), lse=out.get("lse"),
                           argmax=out.get("argmax"), dH=out["dH"], dW=out["dW"],
                           db=out.get("db"), workspace=self.plan.workspace,
                           workspace_bytes=self.plan.workspace_bytes, err_count=out["err"])
        B.fldce_vp_fwd_bwd(self.plan.handle, call, all_stats, all_stats.shape[0])
        return out


def fwd_bwd_vocab_parallel(kernels, H, W_shard, target, p_mask, *, total: float = 0.0,
                           grad_out: float = 1.0, bias_shard=None, out: Optional[dict] = None,
                           group=None) -> dict:
    """One vocabulary-parallel step (the tensor-parallel tutorial page, section 4).

    Every rank holds all tokens (H, target, p_mask) and the rows of W (and
    bias) of its vocabulary shard; ranks are ordered by vocabulary offset.
    1. each rank's sweep 1 writes per-token shard statistics (max, sum-exp,
       target logit, logit sum, argmax): 32 bytes per token;
    2. the statistics are all-gathered; every rank merges them in rank order
       into the same lse and loss, and forms G for its own columns, giving
       its dW and db shard and its partial dH;
    3. the partial dH are summed across ranks.
    Returns this rank's outputs: loss (the job's), dH (summed), dW / db (the
    shard's).  Every rank holds all tokens, so the count normaliser is local.
    """
    stats = kernels.vp_stats(H, W_shard, target, p_mask, bias_shard)
    P = dist.get_world_size(group)
    all_stats = torch.empty((P,) + tuple(stats.shape), dtype=stats.dtype, device=stats.device)
    dist.all_gather([all_stats[r] for r in range(P)], stats.contiguous(), group=group)
    out = kernels.vp_fwd_bwd(H, W_shard, target, p_mask, total, grad_out, bias_shard,
                             all_stats, out)
    dist.all_reduce(out["dH"], op=dist.ReduceOp.SUM, group=group)
    return out
