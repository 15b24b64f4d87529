"""Host-to-host streaming pipeline around one KVCache.

A caller whose chunks' Q, K, V arrive in host memory and whose outputs go
back to the host runs three things per AR step: the upload of q, k, v, the
step itself (evict, append, attend) and the download of the output.  Run one
after another they add up; here they run on three CUDA streams so that step
k's upload overlaps step k-1's compute and step k-2's download, with two
device slots for the inputs and two for the outputs:

  upload stream    H2D q, k, v -> in[s]           after compute of the step that last read in[s]
  compute stream   evict, append, attention       after upload of in[s] and download of out[s]
                   in[s] -> out[s]
  download stream  D2H out[s] -> the caller's     after compute into out[s]
                   host output

(s = step parity).  The ring is host state: each step's evict and slot
assignment happen at submit time and reach the kernels as launch parameters,
so no step waits on the host.  Host buffers must be pinned for the copies to
be asynchronous; the caller must not reuse a host buffer of step k before
``done(k)`` (or ``synchronize``).
"""
from __future__ import annotations

from typing import List, Optional

import torch

from .cache import KVCache


class HostPipeline:
    """streams: optional (upload, compute, download) streams to share with
    other pipelines, e.g. one per layer of a model whose layers must run one
    after another; by default the pipeline creates its own three."""

    def __init__(self, cache: KVCache, streams=None):
        self.cache = cache
        dev = cache.device
        d = cache.desc
        shape = (d.B, cache.Lq, d.H, 128)
        self.inputs = [{n: torch.empty(shape, dtype=torch.bfloat16, device=dev) for n in "qkv"}
                       for _ in range(2)]
        self.outputs = [torch.empty(shape, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        if streams is None:
            streams = tuple(torch.cuda.Stream(dev) for _ in range(3))
        self.up, self.compute, self.down = streams
        ev = lambda: torch.cuda.Event()
        self.uploaded = [ev() for _ in range(2)]
        self.computed = [ev() for _ in range(2)]
        self.downloaded = [ev() for _ in range(2)]
        self.used = [False, False]          # slot has a step in flight
        self.step_events: List[torch.cuda.Event] = []

    def submit(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
               shot: Optional[List[int]] = None) -> int:
        """Queue one AR step: q, k, v pinned host bf16 [B, C*T, H, 128]; out a
        pinned host tensor of the same shape that receives the attention
        output.  shot: optional shot id per stream (kv_ring_begin_shot).
        Returns the step's index for ``done``."""
        s = len(self.step_events) & 1
        c = self.cache
        if shot is not None:
            for b, sid in enumerate(shot):
                c.begin_shot(b, sid)
        need = c.desc.C - min(c.free_frames(b) for b in range(c.desc.B))
        if need > 0:
            c.evict(need)
        dev_in = self.inputs[s]
        with torch.cuda.stream(self.up):
            if self.used[s]:
                self.up.wait_event(self.computed[s])        # step k-2 has read in[s]
            for name, host in (("q", q), ("k", k), ("v", v)):
                dev_in[name].copy_(host, non_blocking=True)
            self.uploaded[s].record(self.up)
        self.compute.wait_event(self.uploaded[s])
        if self.used[s]:
            self.compute.wait_event(self.downloaded[s])     # step k-2's output is home
        c.append(dev_in["k"], dev_in["v"], stream=self.compute)
        c.attention(dev_in["q"], out=self.outputs[s], stream=self.compute)
        self.computed[s].record(self.compute)
        with torch.cuda.stream(self.down):
            self.down.wait_event(self.computed[s])
            out.copy_(self.outputs[s], non_blocking=True)
            self.downloaded[s].record(self.down)
        self.used[s] = True
        done = torch.cuda.Event()
        done.record(self.down)
        self.step_events.append(done)
        return len(self.step_events) - 1

    def done(self, step: int) -> bool:
        return self.step_events[step].query()

    def synchronize(self) -> None:
        for st in (self.up, self.compute, self.down):
            st.synchronize()
