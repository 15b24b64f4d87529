"""Oracle of the sequence-parallel merge (test infrastructure only).

"NVlabs/LongLive 2.0: NVFP4 parallel infrastructure for long video
generation", section "NVFP4, sequence parallel and the async decode path",
names sequence-parallel inference as the way to cut the KV memory each GPU
holds; it does not spell out the split.  Reading: the KV split, each shard
holding a contiguous share of every frame's tokens, each computing the chunk
attention over its own keys, the results combined per query row.

For disjoint key sets K_1 .. K_n with logits s and values v, the softmax
attention over their union is a weighted sum of the per-set attentions:
with Z_j = sum_{k in K_j} exp(s_k), L_j = log Z_j and O_j = sum exp(s_k) v_k
/ Z_j, the union has Z = sum_j Z_j, so L = log sum_j exp(L_j) and
O = sum_j (Z_j / Z) O_j = sum_j exp(L_j - L) O_j.  ``lse_merge`` writes that
out in fp64; an empty set (L_j = -inf) has weight 0.
"""
from __future__ import annotations

import numpy as np


def lse_merge(o_parts, lse_parts):
    """o_parts: n arrays [..., 128]; lse_parts: n arrays [...] (natural log).
    Returns (O [..., 128], L [...]) in fp64."""
    o = np.stack([np.asarray(x, np.float64) for x in o_parts])       # [n, ..., 128]
    lse = np.stack([np.asarray(x, np.float64) for x in lse_parts])    # [n, ...]
    m = lse.max(axis=0)
    finite = np.isfinite(m)
    w = np.where(finite[None], np.exp(lse - np.where(finite, m, 0.0)[None]), 0.0)
    z = w.sum(axis=0)
    safe = np.where(z > 0, z, 1.0)
    out = (w[..., None] * np.where(w[..., None] > 0, o, 0.0)).sum(axis=0) / safe[..., None]
    L = np.where(z > 0, m + np.log(safe), -np.inf)
    return out, L


def shard_tokens(T: int, count: int, rank: int):
    """Token range [t0, t1) of every frame held by shard `rank` of `count`."""
    if count < 1 or T % count or not 0 <= rank < count:
        raise ValueError("T must split evenly into count shards")
    ts = T // count
    return rank * ts, (rank + 1) * ts
