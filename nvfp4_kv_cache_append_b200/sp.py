"""Sequence-parallel KV split across the GPUs of one node.

"NVlabs/LongLive 2.0: NVFP4 parallel infrastructure for long video
generation", section "NVFP4, sequence parallel and the async decode path",
runs inference sequence-parallel to cut the KV memory each GPU holds.  Here
each rank's ``KVCache`` is one shard of the cache: rank r holds tokens
[r*T/n, (r+1)*T/n) of every frame (n ranks, T tokens per frame).  One AR
step on every rank:

  1. evict when full and append the whole chunk's K/V: the shard quantizes
     and stores its own tokens (all ranks run the same ring);
  2. attention of the whole chunk's queries over the shard's keys, with the
     lse, into this rank's half of a double-buffered partial-result buffer in
     symmetric memory (every rank can load every other rank's buffer);
  3. ``nvkv_lse_merge_synced``: one kernel that signals every rank through
     device flags in the same symmetric buffer, waits (bounded) for every
     rank's signal of this step, then merges query rows [r*Lq/n, (r+1)*Lq/n)
     (this rank's slice of the chunk) from all n partial results, n - 1 of
     them read from the peers' memory over NVLink: barrier, exchange and
     merge are one launch.

The rank ends the step with the attention output of its own query slice, the
layout the rest of a sequence-parallel layer works on.  PyTorch provides the
process group and the symmetric allocation; the path runs in libnvkv.so's
kernels.  A barrier wait that runs out writes NVKV_ERR_TIMEOUT to the cache's
status word (``cache.device_status()``) instead of trapping.  The slot of the
partial buffer alternates per step: a rank overwrites slot s only two steps
later, after the barrier of the step in between, which every rank passes only
once it has finished merging from s.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional, Tuple

import torch

from . import _lib as L
from .cache import KVCache, _stream


@dataclass(frozen=True)
class SPPlan:
    """Which tokens and query rows rank ``rank`` of ``world`` owns."""
    rank: int
    world: int
    T: int          # tokens per frame
    Lq: int         # query rows of a chunk (C * T)

    def __post_init__(self):
        if not 0 <= self.rank < self.world or self.T % self.world or self.Lq % self.world:
            raise ValueError("T and Lq must split evenly over the ranks")

    @property
    def tokens(self) -> Tuple[int, int]:
        ts = self.T // self.world
        return self.rank * ts, (self.rank + 1) * ts

    @property
    def queries(self) -> Tuple[int, int]:
        n = self.Lq // self.world
        return self.rank * n, (self.rank + 1) * n


class SequenceParallelKV:
    """This rank's shard of a KV cache split over a process group (one GPU per
    rank, NCCL); ``step`` returns the chunk attention of this rank's query
    slice over the whole cache."""

    FLAG_BYTES = 64          # NVKV_MAX_SHARDS uint32 signals per rank

    def __init__(self, B: int, H: int, grid_h: int, grid_w: int, C: int, S: int, W: int,
                 kv_dtype: int = L.NVKV_KV_NVFP4, group=None, barrier_timeout_ms: int = 10000):
        import torch.distributed as dist
        import torch.distributed._symmetric_memory as symm_mem
        self.group = group if group is not None else dist.group.WORLD
        rank, world = dist.get_rank(self.group), dist.get_world_size(self.group)
        device = torch.device("cuda", torch.cuda.current_device())
        self.cache = KVCache(B, H, grid_h, grid_w, C, S, W, kv_dtype, device=device,
                             shard_rank=rank, shard_count=world)
        self.plan = SPPlan(rank, world, self.cache.T, self.cache.Lq)
        self.B, self.H, self.Lq = B, H, self.cache.Lq
        self.o_bytes = B * self.Lq * H * 128 * 2
        self.l_bytes = B * H * self.Lq * 4
        self.slot_bytes = (self.o_bytes + self.l_bytes + 255) // 256 * 256
        self.buf = symm_mem.empty(2 * self.slot_bytes + self.FLAG_BYTES, dtype=torch.uint8,
                                  device=device)
        self.hdl = symm_mem.rendezvous(self.buf, self.group)
        self.ptrs = list(self.hdl.buffer_ptrs)
        self.flag_ptrs = [p + 2 * self.slot_bytes for p in self.ptrs]
        # every rank's flags are zero before any rank signals
        self.buf[2 * self.slot_bytes:].zero_()
        torch.cuda.synchronize(device)
        dist.barrier(group=self.group)
        self.timeout_ms = barrier_timeout_ms
        self.steps = 0

    def _slot_views(self, s: int):
        base = s * self.slot_bytes
        o = self.buf[base:base + self.o_bytes].view(torch.bfloat16).view(self.B, self.Lq, self.H, 128)
        l = self.buf[base + self.o_bytes:base + self.o_bytes + self.l_bytes].view(torch.float32)
        return o, l.view(self.B, self.H, self.Lq)

    def step(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
             out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """q, k, v: the whole chunk's bf16 [B, C*T, H, 128] (same on every
        rank).  Returns bf16 [B, Lq/world, H, 128]: rows plan.queries."""
        s = self.steps & 1
        self.steps += 1
        o_part, l_part = self._slot_views(s)
        self.cache.step(q, k, v, out=o_part, lse=l_part)
        q0, q1 = self.plan.queries
        if out is None:
            out = torch.empty((self.B, q1 - q0, self.H, 128), dtype=torch.bfloat16, device=q.device)
        elif tuple(out.shape) != (self.B, q1 - q0, self.H, 128) or out.dtype != torch.bfloat16 \
                or not out.is_contiguous():
            raise ValueError(f"out must be contiguous bf16 [{self.B}, {q1 - q0}, {self.H}, 128]")
        base = s * self.slot_bytes
        epoch = self.steps & 0xFFFFFFFF or 1
        L.nvkv_lse_merge_synced([p + base for p in self.ptrs],
                                [p + base + self.o_bytes for p in self.ptrs], self.flag_ptrs,
                                self.plan.rank, epoch, self.timeout_ms * 1000,
                                self.cache.status.data_ptr(), self.B, self.H, self.Lq, q0, q1,
                                out.data_ptr(), None, _stream(None))
        return out
