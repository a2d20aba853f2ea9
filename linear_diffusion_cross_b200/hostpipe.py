"""Host <-> device pipeline for callers whose inputs and results live in host memory.

Each step's inputs (H, W, target, p_mask) are copied from pinned host memory
into one of two device slots on an upload stream, while the fused call of the
previous step runs on the compute stream from the other slot.  Each slot also
owns its own output buffers, so step i's results (loss, dH, dW) can be copied
back to pinned host memory on a download stream while step i+1 computes into
the other slot.  Events order the three streams:

* a slot's inputs are refilled only after the call that read them finished;
* a call starts only after its slot's inputs have landed, and only after the
  download of the results that slot held two steps earlier has finished;
* a download starts only after the call that wrote the results finished --
  except dW's: the library computes the last chunk's dW before its dH and
  records an event as soon as dW is final, and dW (the largest result)
  starts downloading then, while dH is still being computed.

Every step still moves all of its inputs and results; the copies overlap the
neighbouring steps' compute (PCIe upload and download run concurrently on
separate copy engines).  After ``run`` returns, the compute stream is ordered
after the last download, so an event recorded on it afterwards covers every
copy.  PyTorch provides the buffers, streams and events; the computation is
the library's.
"""
from __future__ import annotations

from typing import Iterable, Optional, Sequence

import torch

from . import binding as B

# results a step can hand back to the host
RESULT_KEYS = ("loss", "dH", "dW")


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
                "out": plan.outputs(N, want_rows=False),
            })
        self.copy_stream = torch.cuda.Stream(device=dev)      # host -> device
        self.fetch_stream = torch.cuda.Stream(device=dev)     # device -> host
        self.filled = [torch.cuda.Event() for _ in range(2)]    # inputs landed
        self.done = [torch.cuda.Event() for _ in range(2)]      # the call finished
        self.fetched = [torch.cuda.Event() for _ in range(2)]   # results downloaded
        # dW final (recorded by the library by handle, so created up front)
        self.dw_ready = [torch.cuda.Event() for _ in range(2)]
        cur = torch.cuda.current_stream(dev)
        for e in self.dw_ready:
            e.record(cur)
        self._last = 0

    @property
    def out(self) -> dict:
        """Device outputs of the last step run."""
        return self.slots[self._last]["out"]

    def h2d_bytes(self) -> int:
        s = self.slots[0]
        return sum(s[k].numel() * s[k].element_size() for k in ("H", "W", "y", "p")
                   if s[k] is not None)

    def host_results(self, keys: Sequence[str] = RESULT_KEYS) -> dict:
        """Pinned host buffers shaped like one step's results."""
        o = self.slots[0]["out"]
        return {k: torch.empty(o[k].shape, dtype=o[k].dtype).pin_memory() for k in keys}

    @staticmethod
    def d2h_bytes(results: dict) -> int:
        return sum(t.numel() * t.element_size() for t in results.values())

    def _fill(self, slot: int, host: dict):
        s = self.slots[slot]
        cs = self.copy_stream
        cs.wait_event(self.done[slot])             # the call that read this slot is done
        with torch.cuda.stream(cs):
            s["H"].copy_(host["H"], non_blocking=True)
            s["W"].copy_(host["W"], non_blocking=True)
            s["y"].copy_(host["y"], non_blocking=True)
            if s["p"] is not None and host.get("p") is not None:
                s["p"].copy_(host["p"], non_blocking=True)
        self.filled[slot].record(cs)

    def _compute(self, slot: int, total: float, grad_out: float, stream) -> None:
        s = self.slots[slot]
        stream.wait_event(self.filled[slot])
        stream.wait_event(self.fetched[slot])      # results of two steps ago are out
        self.plan.fwd_bwd(s["H"], s["W"], s["y"], s["p"], total, grad_out, out=s["out"],
                          stream=stream, dw_ready_event=self.dw_ready[slot])
        self.done[slot].record(stream)

    def _fetch(self, slot: int, copies) -> None:
        """Copy (key, host tensor) pairs of the slot's results to the host:
        dW as soon as it is final, the rest once the call has finished."""
        fs = self.fetch_stream
        out = self.slots[slot]["out"]
        early = [(k, t) for k, t in copies if k == "dW"]
        late = [(k, t) for k, t in copies if k != "dW"]
        if early:
            fs.wait_event(self.dw_ready[slot])
            with torch.cuda.stream(fs):
                for k, t in early:
                    t.copy_(out[k], non_blocking=True)
        fs.wait_event(self.done[slot])
        with torch.cuda.stream(fs):
            for k, t in late:
                t.copy_(out[k], non_blocking=True)
        self.fetched[slot].record(fs)

    def run(self, batches: Iterable[dict], total: float, grad_out: float = 1.0,
            stream: Optional[torch.cuda.Stream] = None,
            results: Optional[Sequence[Optional[dict]]] = None) -> torch.Tensor:
        """One step per host batch ({"H", "W", "y", "p"}: pinned CPU tensors).

        ``results``, if given, holds one entry per batch: a dict of pinned
        host tensors (any of "loss", "dH", "dW"; see ``host_results``) that
        receives that step's results, or None.  The same dict may serve
        several steps (a download into it is ordered after the previous one);
        its contents are then the last of those steps'.

        Returns a pinned CPU tensor of the steps' losses.  Everything is
        valid once the compute stream has been synchronised."""
        stream = stream or torch.cuda.current_stream(self.plan.device)
        batches = list(batches)
        if results is not None and len(results) != len(batches):
            raise ValueError("results needs one entry per batch")
        losses = torch.empty(len(batches), dtype=torch.float32).pin_memory()
        if not batches:
            return losses
        # no copy starts before the work already queued on the compute stream
        self.copy_stream.wait_stream(stream)
        self.fetch_stream.wait_stream(stream)
        self._fill(0, batches[0])
        for i in range(len(batches)):
            slot = i % 2
            if i + 1 < len(batches):
                self._fill((i + 1) % 2, batches[i + 1])
            self._compute(slot, total, grad_out, stream)
            copies = [("loss", losses[i:i + 1])]
            if results is not None and results[i] is not None:
                copies += [(k, v) for k, v in results[i].items() if k in RESULT_KEYS]
            self._fetch(slot, copies)
            self._last = slot
        stream.wait_stream(self.fetch_stream)
        return losses
