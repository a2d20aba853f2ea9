"""Host -> device input pipeline for callers whose inputs live in host memory.

Each step's inputs (H, W, target, p_mask) are copied from pinned host memory
into one of two device slots on a copy stream, while the fused call of the
previous step runs on the compute stream from the other slot.  Events order
the two: a slot is refilled only after the call that read it has finished,
and a call starts only after its slot has been filled.  Every step still
moves all of its inputs; the copies just overlap the previous step's
compute.  The loss of each step is copied back to pinned host memory on the
compute stream.  PyTorch provides the buffers, streams and events; the
computation is the library's.
"""
from __future__ import annotations

from typing import Iterable, Optional

import torch

from . import binding as B


class HostPipeline:
    def __init__(self, plan: B.Plan, N: int, *, with_p_mask: bool = True):
        dev = plan.device
        self.plan = plan
        self.N = int(N)
        self.slots = []
        for _ in range(2):
            self.slots.append({
                "H": torch.empty(N, plan.D, dtype=plan.dtype, device=dev),
                "W": torch.empty(plan.V, plan.D, dtype=plan.dtype, device=dev),
                "y": torch.empty(N, dtype=torch.int64, device=dev),
                "p": torch.empty(N, dtype=torch.float32, device=dev) if with_p_mask else None,
            })
        self.copy_stream = torch.cuda.Stream(device=dev)
        self.filled = [torch.cuda.Event() for _ in range(2)]
        self.freed = [torch.cuda.Event() for _ in range(2)]
        self.out = plan.outputs(N, want_rows=False)

    def h2d_bytes(self) -> int:
        s = self.slots[0]
        return sum(t.numel() * t.element_size() for t in s.values() if t is not None)

    def _fill(self, slot: int, host: dict):
        s = self.slots[slot]
        cs = self.copy_stream
        cs.wait_event(self.freed[slot])            # the call that read this slot is done
        with torch.cuda.stream(cs):
            s["H"].copy_(host["H"], non_blocking=True)
            s["W"].copy_(host["W"], non_blocking=True)
            s["y"].copy_(host["y"], non_blocking=True)
            if s["p"] is not None and host.get("p") is not None:
                s["p"].copy_(host["p"], non_blocking=True)
        self.filled[slot].record(cs)

    def _compute(self, slot: int, total: float, grad_out: float, stream,
                 loss_host: torch.Tensor) -> None:
        s = self.slots[slot]
        stream.wait_event(self.filled[slot])
        self.plan.fwd_bwd(s["H"], s["W"], s["y"], s["p"], total, grad_out, out=self.out,
                          stream=stream)
        self.freed[slot].record(stream)
        with torch.cuda.stream(stream):
            loss_host.copy_(self.out["loss"], non_blocking=True)

    def run(self, batches: Iterable[dict], total: float, grad_out: float = 1.0,
            stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """One step per host batch ({"H", "W", "y", "p"}: pinned CPU tensors).
        Returns a pinned CPU tensor of the steps' losses, valid once the
        compute stream has been synchronised; dH / dW of the last step are in
        ``self.out``."""
        stream = stream or torch.cuda.current_stream(self.plan.device)
        batches = list(batches)
        losses = torch.empty(len(batches), dtype=torch.float32).pin_memory()
        if not batches:
            return losses
        # no copy starts before the work already queued on the compute stream
        self.copy_stream.wait_stream(stream)
        self._fill(0, batches[0])
        for i in range(len(batches)):
            if i + 1 < len(batches):
                self._fill((i + 1) % 2, batches[i + 1])
            self._compute(i % 2, total, grad_out, stream, losses[i:i + 1])
        return losses
