"""Oracle model of the sink + rolling-window KV ring (test infrastructure only).

Follows "NVlabs/LongLive 2.0: NVFP4 parallel infrastructure for long video
generation", section "NVFP4, sequence parallel and the async decode path"
(attention sink; multi-shot attention sink) and "LongLive: NVIDIA long video
generation" (evermx.com), heading "Multi-Shot Generation", with the cache
contract of the streaming workloads:

  * capacity is S + W frames; the window holds the current chunk too;
  * the first S frames appended are the global sink and are never evicted;
  * eviction drops the oldest non-sink, unpinned frames;
  * logical order = sink frames first, then the other resident frames by age;
    a key frame's RoPE frame index is its rank in that order (masked frames
    included), and a query frame's index is the rank of its own keys;
  * multi-shot: the first chunk of shot s > 0 is pinned in the window while
    shot s runs (unpinned when shot s+1 begins).  A chunk of shot s sees the
    global sink, every frame of shot s, and, of earlier shots, only each
    shot's last frame.

This model tracks frame identities only (no physical slots, no data).
"""
from __future__ import annotations

import dataclasses
from typing import List


@dataclasses.dataclass
class Frame:
    fid: int          # global frame index (0, 1, 2, ... in append order)
    shot: int
    sink: bool
    pinned: bool
    shot_last: bool   # last frame of a shot that has ended


class OracleRing:
    def __init__(self, S: int, W: int, C: int):
        self.S, self.W, self.C = S, W, C
        self.frames: List[Frame] = []
        self.next_fid = 0
        self.shot = 0
        self.pin_next = False

    @property
    def capacity(self) -> int:
        return self.S + self.W

    def n_evictable(self) -> int:
        return sum(1 for f in self.frames if not f.sink and not f.pinned)

    def evict(self, n: int) -> List[int]:
        """Drop the n oldest evictable frames; returns their frame indices."""
        if n > self.n_evictable():
            raise ValueError("not enough evictable frames")
        gone = []
        keep = []
        for f in self.frames:
            if len(gone) < n and not f.sink and not f.pinned:
                gone.append(f.fid)
            else:
                keep.append(f)
        self.frames = keep
        return gone

    def begin_shot(self, shot: int) -> None:
        if shot == self.shot:
            return
        if shot < self.shot:
            raise ValueError("shots only move forward")
        if self.frames:
            self.frames[-1].shot_last = True
        for f in self.frames:
            f.pinned = False
        self.shot = shot
        self.pin_next = shot > 0

    def append(self) -> List[int]:
        """Append one chunk (C frames); returns their frame indices."""
        if len(self.frames) + self.C > self.capacity:
            raise ValueError("ring full: evict first")
        new = []
        for _ in range(self.C):
            fid = self.next_fid
            self.next_fid += 1
            self.frames.append(Frame(fid, self.shot, sink=fid < self.S, pinned=self.pin_next,
                                     shot_last=False))
            new.append(fid)
        self.pin_next = False
        return new

    def step(self) -> List[int]:
        """One AR step's cache update: evict when full, then append."""
        need = len(self.frames) + self.C - self.capacity
        if need > 0:
            self.evict(need)
        return self.append()

    # ---------------------------------------------------------- read side

    def resident(self) -> List[int]:
        return [f.fid for f in self.frames]

    def visible(self):
        """[(frame index, RoPE frame position)] seen by the newest chunk."""
        out = []
        for rank, f in enumerate(self.frames):
            if f.sink or f.shot == self.shot or f.shot_last:
                out.append((f.fid, rank))
        return out

    def query_pos0(self) -> int:
        """RoPE frame position of the newest chunk's first frame."""
        return len(self.frames) - self.C
