"""Test helpers: drive the CUDA library and the oracle on the same seeded inputs.

Parity bars (stated by the workload contract): packed codes and scale bytes
bit-exact; attention outputs within max-abs 3e-2 and relative L2 1e-2 of the
fp64 oracle run on the same dequantized K/V and bf16 Q.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import kvsynth

TOL_MAX_ABS = 3e-2
TOL_REL_L2 = 1e-2


def parity(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    d = got - ref
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))
    return max_abs, rel


def assert_parity(got, ref, what=""):
    max_abs, rel = parity(got, ref)
    log = os.environ.get("NVKV_PARITY_LOG")
    if log:
        with open(log, "a") as f:
            f.write(json.dumps({"case": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0],
                                "what": what, "max_abs": max_abs, "rel_l2": rel}) + "\n")
    assert np.isfinite(got).all(), what
    assert max_abs <= TOL_MAX_ABS and rel <= TOL_REL_L2, f"{what}: max_abs {max_abs:.3e} rel_l2 {rel:.3e}"
    return max_abs, rel


class LibStream:
    """The CUDA path for one workload: KVCache + shot schedule, one AR step per call."""

    def __init__(self, wl: kvsynth.Workload, kv_dtype: int, sched=None, seed: int = 0):
        import nvfp4_kv_cache_append_b200 as nv
        self.nv = nv
        self.wl = wl
        self.cache = nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, kv_dtype)
        self.sched = sched if sched is not None else kvsynth.shot_schedule(wl, seed)
        self.step_no = 0

    def step(self, q, k, v, with_lse=True):
        self.step_no += 1
        for b in range(self.wl.B):
            self.cache.begin_shot(b, self.sched[b][self.step_no - 1])
        lse = None
        if with_lse:
            lse = torch.empty(self.wl.B, self.wl.H, self.wl.Lq, dtype=torch.float32,
                              device=q.device)
        out = self.cache.step(q, k, v, lse=lse)
        return out, lse

    def frame_slot(self, b: int, fid: int) -> int:
        st = self.cache.ring.s[b]
        for i in range(st.n_resident):
            if st.frame[i] == fid:
                return st.slot[i]
        raise KeyError(fid)

    def frame_rows(self, b: int, fid: int):
        T = self.wl.T
        p = self.frame_slot(b, fid)
        return slice(p * T, (p + 1) * T)


def to_gpu(x: dict):
    return {k: v.cuda() for k, v in x.items()}


def sample_rows(Lq: int, n_random: int, seed: int):
    """Query rows spanning Q tiles: tile edges, the ragged tail, random picks."""
    fixed = {0, 1, 63, 64, 127, 128, 129, Lq // 2, Lq - 129, Lq - 128, Lq - 1}
    rows = sorted(r for r in fixed if 0 <= r < Lq)
    rng = np.random.default_rng(seed)
    rows += rng.choice(Lq, size=min(n_random, Lq), replace=False).tolist()
    return np.unique(np.array(rows, np.int64))
