"""Streaming oracle: the whole AR loop on the CPU (test infrastructure only).

One AR step is append-then-attend (reading: a step quantizes the new chunk's
K/V with the per-head global scale fixed by step 1, appends it to the sink +
window ring, then the chunk's queries attend over every visible cached frame,
their own frames included).  Keys are cached before RoPE and rotated at read
time, following "NVlabs LongLive" (refft.com), Core Analysis block "How do
KV-cache relative RoPE and TriAttention work together".

With ``fp4_qk=True`` the stream follows the block-scaled FP4 Q K^T reading
(``nvfp4_oracle.c``, section "block-scaled FP4 Q K^T (a reading)"): K is
cached with its spatial RoPE applied before quantization and the logits are
taken between FP4 Q (rotated per key frame) and the cached FP4 K.

Inputs come from ``kvsynth`` only; no value comes from the CUDA path.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Tuple

import numpy as np

import kvsynth
from . import (amax as _amax, attention_rows, attention_rows_fp4qk, dequant_rows, global_scale,
               k_spatial_rope_f32, quantize_rows)
from .ring import OracleRing


class OracleStream:
    def __init__(self, wl: kvsynth.Workload, seed: int = 0,
                 shot_sched: Optional[List[List[int]]] = None, keep_inputs: bool = True,
                 fp4_qk: bool = False):
        self.wl = wl
        self.fp4_qk = fp4_qk
        self.seed = seed
        self.rings = [OracleRing(wl.S, wl.W, wl.C) for _ in range(wl.B)]
        self.sched = shot_sched if shot_sched is not None else kvsynth.shot_schedule(wl, seed)
        self.s_g: Optional[np.ndarray] = None      # [2, B, H] float32 (K, V)
        self.store: Dict[Tuple[int, int], dict] = {}
        self.step_no = 0
        self.keep_inputs = keep_inputs
        self.q = None                              # bf16 Q of the current step

    # ------------------------------------------------------------ append

    def _k_rows(self, kf, b, h, sl=None):
        """K rows [n, 128] of (b, h) over chunk rows ``sl`` as the cache
        quantizes them: as given, or spatially rotated (``fp4_qk``)."""
        wl = self.wl
        sl = slice(0, wl.Lq) if sl is None else sl
        rows = np.ascontiguousarray(kf[b, sl, h, :])
        if not self.fp4_qk:
            return rows
        tok = (np.arange(wl.Lq, dtype=np.int32) % wl.T)[sl]
        return k_spatial_rope_f32(rows, tok, wl.grid_w)

    def _scales_from(self, k, v) -> np.ndarray:
        wl = self.wl
        s = np.zeros((2, wl.B, wl.H), np.float32)
        kf, vf = k.float().numpy(), v.float().numpy()
        for b in range(wl.B):
            for h in range(wl.H):
                s[0, b, h] = global_scale(_amax(self._k_rows(kf, b, h)))
                s[1, b, h] = global_scale(_amax(np.ascontiguousarray(vf[b, :, h, :])))
        return s

    def step(self, k=None, v=None, q=None):
        """Advance one AR step; returns {b: [new frame indices]}."""
        wl = self.wl
        self.step_no += 1
        if k is None or v is None or q is None:
            x = kvsynth.chunk_qkv(wl, self.step_no, self.seed)
            k, v, q = x["k"], x["v"], x["q"]
        self.q = q
        if self.step_no == 1:
            self.s_g = self._scales_from(k, v)
        new = {}
        kf = k.float().numpy()
        vf = v.float().numpy()
        for b, ring in enumerate(self.rings):
            ring.begin_shot(self.sched[b][self.step_no - 1])
            need = len(ring.frames) + wl.C - ring.capacity
            if need > 0:
                for fid in ring.evict(need):
                    self.store.pop((b, fid), None)
            fids = ring.append()
            self._store_chunk(b, fids, kf, vf)
            new[b] = fids
        return new

    def overwrite(self, k, v, q):
        """A denoising step inside the current AR step: the newest chunk's K/V
        replaced in place, ring unchanged (the pages' in-place quantized
        KV-cache update, "NVlabs/LongLive 2.0: NVFP4 parallel infrastructure
        for long video generation", section "NVFP4, sequence parallel and the
        async decode path").  Reading: while the first chunk is the only
        chunk appended, its global scales are fixed again from the new
        values, since they are defined by the first chunk; afterwards they
        stay fixed.  Returns {b: [the chunk's frame indices]}."""
        wl = self.wl
        if self.step_no < 1:
            raise ValueError("no chunk appended yet")
        self.q = q
        if self.step_no == 1:
            self.s_g = self._scales_from(k, v)
        kf = k.float().numpy()
        vf = v.float().numpy()
        new = {}
        for b, ring in enumerate(self.rings):
            fids = list(range(ring.next_fid - wl.C, ring.next_fid))
            self._store_chunk(b, fids, kf, vf)
            new[b] = fids
        return new

    def _store_chunk(self, b, fids, kf, vf):
        """Quantize the chunk's frames of stream b (quantize_rows per head)."""
        wl = self.wl
        for c, fid in enumerate(fids):
            sl = slice(c * wl.T, (c + 1) * wl.T)
            ent = {}
            for name, xf, t in (("k", kf, 0), ("v", vf, 1)):
                rows = np.ascontiguousarray(xf[b, sl].transpose(1, 0, 2))   # [H, T, D]
                codes = np.zeros((wl.H, wl.T, 64), np.uint8)
                scales = np.zeros((wl.H, wl.T, 8), np.uint8)
                for h in range(wl.H):
                    src = self._k_rows(kf, b, h, sl) if name == "k" else rows[h]
                    codes[h], scales[h] = quantize_rows(src, self.s_g[t, b, h])
                ent[name + "_codes"] = codes
                ent[name + "_scales"] = scales
                if self.keep_inputs:
                    ent[name + "_bf16"] = rows
            self.store[(b, fid)] = ent

    # ------------------------------------------------------------- read

    def frame(self, b: int, fid: int) -> dict:
        return self.store[(b, fid)]

    def visible_kv(self, b: int, h: int, quantized: bool = True, tokens=None):
        """Visible keys/values of the newest chunk for (b, h) in logical order.

        Returns (k [Lk,128] f64, v [Lk,128] f64, k_frame_pos [Lk], k_tok [Lk]).
        ``quantized=False`` gives the bf16 cache (the bf16-KV twin);
        ``tokens=(t0, t1)`` keeps tokens t0 .. t1-1 of every frame (one shard
        of a sequence-parallel KV split, ``oracle.merge``)."""
        wl = self.wl
        t0, t1 = (0, wl.T) if tokens is None else tokens
        ks, vs, fpos, tok = [], [], [], []
        for fid, rank in self.rings[b].visible():
            e = self.store[(b, fid)]
            if quantized:
                ks.append(dequant_rows(e["k_codes"][h][t0:t1], e["k_scales"][h][t0:t1],
                                       self.s_g[0, b, h]))
                vs.append(dequant_rows(e["v_codes"][h][t0:t1], e["v_scales"][h][t0:t1],
                                       self.s_g[1, b, h]))
            else:
                ks.append(e["k_bf16"][h][t0:t1].astype(np.float64))
                vs.append(e["v_bf16"][h][t0:t1].astype(np.float64))
            fpos.append(np.full(t1 - t0, rank, np.int32))
            tok.append(np.arange(t0, t1, dtype=np.int32))
        if not ks:
            z = np.zeros((0, 128))
            return z, z, np.zeros(0, np.int32), np.zeros(0, np.int32)
        return np.concatenate(ks), np.concatenate(vs), np.concatenate(fpos), np.concatenate(tok)

    def query_positions(self, b: int):
        wl = self.wl
        l = np.arange(wl.Lq)
        return (self.rings[b].query_pos0() + l // wl.T).astype(np.int32), (l % wl.T).astype(np.int32)

    def attention(self, b: int, h: int, rows, quantized: bool = True, tokens=None):
        """Oracle outputs (fp64) for query rows ``rows`` of (b, h) at the current
        step: (out [n, 128], lse [n]); ``tokens`` as in ``visible_kv``."""
        qpos, qtok = self.query_positions(b)
        q = self.q[b, :, h, :]
        if self.fp4_qk and quantized:
            k, v, fpos, _ = self.visible_kv(b, h, True, tokens)     # K' dequantized
            return attention_rows_fp4qk(q, k, v, fpos, qpos, qtok, rows, self.wl.grid_w)
        k, v, fpos, tok = self.visible_kv(b, h, quantized, tokens)
        return attention_rows(q, k, v, fpos, tok, qpos, qtok, rows, self.wl.grid_w)
