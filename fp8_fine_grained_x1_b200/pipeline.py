"""Steps fed from, and drained to, pinned host memory with the copies
overlapped.

A step (linear.FpropStep, DgradStep, WgradStep, WgradCachedStep, MoeStep)
reads its device inputs (`step.inputs`) and writes `step.output`.  When the
batches live in host memory, the PCIe copies dominate: a dense-MLP Fprop step
moves 323 MB in and 151 MB out for 0.7 ms of GPU work.  HostPipeline keeps
`depth` copies of the step (each with its own device buffers) and three CUDA
streams, so the host->device copy of batch i+1, the compute of batch i and the
device->host copy of result i-1 run at the same time.  PCIe is full duplex,
so a step then costs about the larger of its two copies rather than their sum.

Ordering, per slot s = i % depth (events, no host synchronisation):
  copy-in  of batch i     waits for the compute of batch i - depth (same inputs)
  compute  of batch i     waits for its copy-in and for the copy-out of
                          result i - depth (same output buffer)
  copy-out of result i    waits for its compute
"""
from __future__ import annotations

from typing import Iterable, List, Sequence, Tuple

import torch


class HostPipeline:
    def __init__(self, steps: Sequence, device=None):
        if len(steps) < 2:
            raise ValueError("HostPipeline needs at least two step copies to overlap")
        self.steps = list(steps)
        dev = torch.device(device) if device is not None else self.steps[0].output.device
        self.copy_in = torch.cuda.Stream(dev)
        self.compute = torch.cuda.Stream(dev)
        self.copy_out = torch.cuda.Stream(dev)
        n = len(self.steps)
        self._in_ready = [torch.cuda.Event() for _ in range(n)]
        self._computed = [torch.cuda.Event() for _ in range(n)]
        self._out_done = [torch.cuda.Event() for _ in range(n)]

    def run(self, batches: Iterable[Tuple[List[torch.Tensor], torch.Tensor]]) -> None:
        """Enqueue every (pinned host inputs, pinned host output) batch.  Returns
        without waiting; the results are in the host outputs once the device is
        synchronised (or once `self.copy_out` is)."""
        n = len(self.steps)
        for i, (host_in, host_out) in enumerate(batches):
            s = i % n
            step = self.steps[s]
            if len(host_in) != len(step.inputs):
                raise ValueError(f"batch {i}: {len(host_in)} inputs, step takes {len(step.inputs)}")
            self.copy_in.wait_event(self._computed[s])
            with torch.cuda.stream(self.copy_in):
                for h, d in zip(host_in, step.inputs):
                    d.copy_(h.view(d.shape), non_blocking=True)
            self._in_ready[s].record(self.copy_in)
            self.compute.wait_event(self._in_ready[s])
            self.compute.wait_event(self._out_done[s])
            with torch.cuda.stream(self.compute):
                step(self.compute)
            self._computed[s].record(self.compute)
            self.copy_out.wait_event(self._computed[s])
            with torch.cuda.stream(self.copy_out):
                host_out.copy_(step.output, non_blocking=True)
            self._out_done[s].record(self.copy_out)
