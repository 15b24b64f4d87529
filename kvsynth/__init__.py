"""Seeded synthetic inputs for the NVFP4 KV-cache path.

This module is shared by the CUDA path's tests/benchmark and by the oracle.
It holds workload shapes and random draws only: none of the method's
arithmetic (no quantization, no RoPE, no attention).

Recipe (the streaming workloads of the 1.3B-like and 5B-like generators on
"LongLive: NVIDIA long video generation" (evermx.com), heading "Model Range and
Hardware Requirements", with the shapes fixed by the workload contract):
  * Q, K, V are bf16, drawn as float32 N(0, 1) from a seeded CPU
    ``torch.Generator`` and rounded to bf16 (round-to-nearest-even).
  * In K, 1% of the H*D channels (round(0.01*H*D), at least 1, drawn once per
    run from the seed) are multiplied by 8 (exact in bf16).
  * Every (step, tensor) pair has its own generator seed, so any step's
    inputs can be regenerated without replaying earlier steps.
  * Multi-shot batches: batch 0 uses shots of (8, 8, 8) chunks; each batch
    b > 0 uses (8 + d1, 8 - d1 + d2, 8 - d2) with d1, d2 uniform in {-3..3}.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List

import torch

__all__ = ["Workload", "WORKLOADS", "mix_seed", "outlier_channels", "chunk_qkv",
           "shot_lengths", "shot_schedule"]

TENSOR_Q, TENSOR_K, TENSOR_V, TENSOR_OUTLIER, TENSOR_SHOTS = 0, 1, 2, 3, 4


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    D: int
    grid_h: int
    grid_w: int
    C: int          # frames per chunk
    S: int          # sink frames
    W: int          # local window frames (the current chunk included)
    steps: int      # AR steps the workload runs
    shots: int = 1  # shots per batch element (multi-shot workload)
    chunks_per_shot: int = 0

    @property
    def T(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def Lq(self) -> int:
        return self.C * self.T

    @property
    def capacity_frames(self) -> int:
        return self.S + self.W


WORKLOADS: Dict[str, Workload] = {
    # tiny parity case: 6 AR steps of append-then-attend
    "tiny": Workload("tiny", B=1, H=2, D=128, grid_h=8, grid_w=8, C=1, S=1, W=3, steps=6),
    # 1.3B-like streaming step: 4680 query tokens, 32760 keys per query
    "stream1p3b": Workload("stream1p3b", B=1, H=12, D=128, grid_h=30, grid_w=52, C=3, S=3,
                           W=18, steps=8),
    # 5B-like streaming step: 2640 query tokens, 21120 keys per query
    "stream5b": Workload("stream5b", B=1, H=24, D=128, grid_h=22, grid_w=40, C=3, S=3, W=21,
                         steps=9),
    # long streaming run: 1.3B-like shapes for 600 AR steps
    "long600": Workload("long600", B=1, H=12, D=128, grid_h=30, grid_w=52, C=3, S=3, W=18,
                        steps=600),
    # multi-shot batched: 4 streams, 3 shots of (about) 8 chunks each
    "multishot": Workload("multishot", B=4, H=12, D=128, grid_h=30, grid_w=52, C=3, S=3, W=18,
                          steps=24, shots=3, chunks_per_shot=8),
}


def mix_seed(*parts: int) -> int:
    """splitmix64 over the parts; returns a non-negative 63-bit seed."""
    mask = (1 << 64) - 1
    h = 0x9E3779B97F4A7C15
    for p in parts:
        h = (h ^ (int(p) & mask)) & mask
        h = (h + 0x9E3779B97F4A7C15) & mask
        z = h
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & mask
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & mask
        h = z ^ (z >> 31)
    return h & ((1 << 63) - 1)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def outlier_channels(wl: Workload, seed: int = 0) -> torch.Tensor:
    """Flattened (h * D + d) indices of the K channels scaled by 8."""
    n = max(1, round(0.01 * wl.H * wl.D))
    perm = torch.randperm(wl.H * wl.D, generator=_gen(mix_seed(seed, TENSOR_OUTLIER)))
    return torch.sort(perm[:n]).values


def chunk_qkv(wl: Workload, step: int, seed: int = 0, which: str = "qkv") -> Dict[str, torch.Tensor]:
    """Q, K, V of AR step ``step`` (1-based) as bf16 CPU tensors [B, Lq, H, D]."""
    shape = (wl.B, wl.Lq, wl.H, wl.D)
    out = {}
    for name, tid in (("q", TENSOR_Q), ("k", TENSOR_K), ("v", TENSOR_V)):
        if name not in which:
            continue
        x = torch.randn(shape, generator=_gen(mix_seed(seed, step, tid)), dtype=torch.float32)
        x = x.to(torch.bfloat16)
        if name == "k":
            idx = outlier_channels(wl, seed)
            flat = x.view(wl.B, wl.Lq, wl.H * wl.D)
            flat[:, :, idx] = flat[:, :, idx] * 8
        out[name] = x
    return out


def shot_lengths(wl: Workload, seed: int = 0) -> List[List[int]]:
    """Chunks per shot for each batch element of a multi-shot workload."""
    if wl.shots <= 1:
        return [[wl.steps] for _ in range(wl.B)]
    g = _gen(mix_seed(seed, TENSOR_SHOTS))
    out = []
    base = wl.chunks_per_shot
    for b in range(wl.B):
        if b == 0:
            out.append([base] * wl.shots)
            continue
        d = torch.randint(-3, 4, (wl.shots - 1,), generator=g).tolist()
        lens = []
        prev = 0
        for s in range(wl.shots):
            cur = d[s] if s < wl.shots - 1 else 0
            lens.append(base - prev + cur)
            prev = cur
        out.append(lens)
    return out


def shot_schedule(wl: Workload, seed: int = 0) -> List[List[int]]:
    """shot id of every AR step (0-based step index) for each batch element."""
    sched = []
    for lens in shot_lengths(wl, seed):
        ids = []
        for s, n in enumerate(lens):
            ids += [s] * n
        sched.append(ids[: wl.steps] + [len(lens) - 1] * max(0, wl.steps - len(ids)))
    return sched
