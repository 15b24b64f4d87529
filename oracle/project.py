"""Oracle of the K/V projection that precedes the append (test
infrastructure only).

The projection maps the chunk's hidden states to keys and values,
K = x W_k^T and V = x W_v^T, and hands bf16 K/V to the append ("NVlabs/
LongLive 2.0: NVFP4 parallel infrastructure for long video generation",
section "NVFP4, sequence parallel and the async decode path": the KV cache
is filled in place from the generator's projections).  Reading: the product
is formed exactly (fp64 here: every bf16 x bf16 product is exact, and the
sums' fp64 rounding lies far below the bf16 rounding that follows), rounded
to fp32 and then to bf16, each to nearest even.  A GPU sums in fp32 in its
own order, so the two agree exactly when every partial sum is an fp32 value
(small-integer inputs, as the exact tests use) and otherwise up to a rare
1-ulp bf16 difference.
"""
from __future__ import annotations

import numpy as np


def bf16_rne(a) -> np.ndarray:
    """fp32 -> bf16 (round to nearest, ties to even), returned as fp32 values."""
    a = np.ascontiguousarray(a, np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    nan = np.isnan(a)
    out = r.astype(np.uint32).view(np.float32)
    return np.where(nan, a, out)


def kv_project(x, w) -> np.ndarray:
    """x [M, hidden], w [N, hidden] (bf16 values) -> bf16(fl32(x w^T)) [M, N] as fp32."""
    y = np.asarray(x, np.float64) @ np.asarray(w, np.float64).T
    return bf16_rne(y.astype(np.float32))
