"""Caller-side plumbing around the C ABI: device planes allocated once with
PyTorch (sizes from ``nvkv_plane_bytes``), the host ring, and one method per
entry point.  PyTorch provides memory and streams only; every step of the
path runs in libnvkv.so's kernels.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _lib as L


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


class KVCache:
    """One sink + rolling-window KV ring (NVFP4 or bf16) on one CUDA device.

    With ``shard_count > 1`` it is shard ``shard_rank`` of a sequence-parallel
    KV split: it holds tokens [rank*T/count, (rank+1)*T/count) of every frame,
    takes whole chunks in ``append``/``attention`` and returns the attention
    over its own keys (merge the shards' results with ``lse_merge``)."""

    def __init__(self, B: int, H: int, grid_h: int, grid_w: int, C: int, S: int, W: int,
                 kv_dtype: int = L.NVKV_KV_NVFP4, device="cuda", shard_rank: int = 0,
                 shard_count: int = 1):
        self.desc = L.nvkv_desc_init(B, H, grid_h, grid_w, C, S, W, kv_dtype)
        if shard_count != 1 or shard_rank != 0:
            L.nvkv_desc_set_shard(self.desc, shard_rank, shard_count)
        self.ring = L.nvkv_ring_init(self.desc)
        self.device = torch.device(device)
        if self.device.type != "cuda":
            raise ValueError("the cache lives in CUDA device memory")
        nb = lambda p: L.nvkv_plane_bytes(self.desc, p)
        alloc = lambda n: torch.zeros(max(n, 16), dtype=torch.uint8, device=self.device)
        self.k_data = alloc(nb(L.NVKV_PLANE_K_DATA))
        self.v_data = alloc(nb(L.NVKV_PLANE_V_DATA))
        fp4 = kv_dtype == L.NVKV_KV_NVFP4
        self.k_scales = alloc(nb(L.NVKV_PLANE_K_SCALES)) if fp4 else None
        self.v_scales = alloc(nb(L.NVKV_PLANE_V_SCALES)) if fp4 else None
        self.amax = alloc(nb(L.NVKV_PLANE_AMAX)) if fp4 else None
        self.s_g = alloc(nb(L.NVKV_PLANE_SCALE_G)) if fp4 else None
        self.status = alloc(nb(L.NVKV_PLANE_STATUS))
        ws = L.nvkv_attention_workspace_bytes(self.desc)
        self.workspace = alloc(ws) if ws else None
        self.ws_bytes = ws
        self.cache = L.nvkv_cache(
            _ptr(self.k_data).value, _ptr(self.v_data).value,
            None if self.k_scales is None else self.k_scales.data_ptr(),
            None if self.v_scales is None else self.v_scales.data_ptr(),
            None if self.amax is None else self.amax.data_ptr(),
            None if self.s_g is None else self.s_g.data_ptr(),
            self.status.data_ptr())
        self.fp4 = fp4

    # ---------------------------------------------------------------- shape
    @property
    def T(self) -> int:
        return self.desc.grid_h * self.desc.grid_w

    @property
    def Ts(self) -> int:
        """Cached tokens of each frame (all T unless this is a shard)."""
        return self.T // self.desc.shard_count

    @property
    def Tr(self) -> int:
        """Rows of each frame slot: Ts, plus one padding row when Ts is odd."""
        return (self.Ts + 1) // 2 * 2

    @property
    def tok_off(self) -> int:
        """Index within the frame of the first cached token."""
        return self.desc.shard_rank * self.Ts

    @property
    def Lq(self) -> int:
        return self.desc.C * self.T

    @property
    def rows(self) -> int:
        return (self.desc.S + self.desc.W) * self.Tr

    def footprint_bytes(self) -> int:
        ts = [self.k_data, self.v_data, self.k_scales, self.v_scales, self.amax, self.s_g,
              self.status, self.workspace]
        return sum(t.numel() * t.element_size() for t in ts if t is not None)

    # ---------------------------------------------------------------- views
    def codes(self, which: str) -> torch.Tensor:
        """[B, H, R, 64] u8 codes (NVFP4) or [B, H, R, 128] bf16 (twin)."""
        t = self.k_data if which == "k" else self.v_data
        d = self.desc
        if self.fp4:
            return t[: d.B * d.H * self.rows * 64].view(d.B, d.H, self.rows, 64)
        return t.view(torch.bfloat16)[: d.B * d.H * self.rows * 128].view(d.B, d.H, self.rows, 128)

    def scales(self, which: str) -> torch.Tensor:
        t = self.k_scales if which == "k" else self.v_scales
        d = self.desc
        return t[: d.B * d.H * self.rows * 8].view(d.B, d.H, self.rows, 8)

    def global_scales(self) -> torch.Tensor:
        return self.s_g.view(torch.float32)[: 2 * self.desc.B * self.desc.H].view(
            2, self.desc.B, self.desc.H)

    def device_status(self) -> int:
        return int(self.status.view(torch.int32)[0].item())

    # -------------------------------------------------------------- entries
    def evict(self, n_frames: int) -> None:
        L.kv_ring_evict(self.desc, self.ring, n_frames)

    def begin_shot(self, b: int, shot_id: int) -> None:
        L.kv_ring_begin_shot(self.desc, self.ring, b, shot_id)

    def visible(self, b: int):
        return L.nvkv_ring_visible(self.desc, self.ring, b)

    def free_frames(self, b: int = 0) -> int:
        return self.desc.S + self.desc.W - self.ring.s[b].n_resident

    def append(self, k: torch.Tensor, v: torch.Tensor, stream=None) -> None:
        self._check_io(k)
        self._check_io(v)
        fn = L.nvfp4_kv_append if self.fp4 else L.bf16_kv_append
        fn(self.desc, self.cache, self.ring, _ptr(k), _ptr(v), _stream(stream))

    def append_spatial_rope(self, k: torch.Tensor, v: torch.Tensor, stream=None) -> None:
        """Quantize-append with K's spatial RoPE applied first (the cache layout
        of the block-scaled FP4 Q K^T reading; see nvfp4_kv_append_spatial_rope)."""
        if not self.fp4:
            raise ValueError("the spatial-RoPE append fills an NVFP4 cache")
        self._check_io(k)
        self._check_io(v)
        L.nvfp4_kv_append_spatial_rope(self.desc, self.cache, self.ring, _ptr(k), _ptr(v),
                                       _stream(stream))

    def overwrite(self, k: torch.Tensor, v: torch.Tensor, stream=None) -> None:
        """Denoising step: the newest chunk's K/V replaced in place (same slots)."""
        self._check_io(k)
        self._check_io(v)
        fn = L.nvfp4_kv_overwrite if self.fp4 else L.bf16_kv_overwrite
        fn(self.desc, self.cache, self.ring, _ptr(k), _ptr(v), _stream(stream))

    def project(self, x: torch.Tensor, w_k: torch.Tensor, w_v: torch.Tensor, k_out=None,
                v_out=None, stream=None):
        """K/V projection on the tensor cores: (x W_k^T, x W_v^T) rounded to
        bf16.  x: bf16 [B, C*T, hidden]; w_k, w_v: bf16 [H*128, hidden]."""
        hidden = self._check_proj(x, w_k, w_v)
        k_out = torch.empty((self.desc.B, self.Lq, self.desc.H, 128), dtype=torch.bfloat16,
                            device=x.device) if k_out is None else k_out
        v_out = torch.empty_like(k_out) if v_out is None else v_out
        self._check_io(k_out)
        self._check_io(v_out)
        L.nvkv_kv_project(self.desc, _ptr(x), hidden, _ptr(w_k), _ptr(w_v), _ptr(k_out),
                          _ptr(v_out), _ptr(self.status), _stream(stream))
        return k_out, v_out

    def project_append(self, x: torch.Tensor, w_k: torch.Tensor, w_v: torch.Tensor,
                       stream=None) -> None:
        """Projection with the NVFP4 quantize-append fused into its epilogue
        (the same cache contents as project + append)."""
        if not self.fp4:
            raise ValueError("the fused projection-append writes an NVFP4 cache")
        hidden = self._check_proj(x, w_k, w_v)
        scratch, nbytes = None, 0
        if not self.ring.scales_fixed:
            nbytes = 2 * self.desc.B * self.Lq * self.desc.H * 128 * 2
            scratch = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
        L.nvfp4_kv_project_append(self.desc, self.cache, self.ring, _ptr(x), hidden, _ptr(w_k),
                                  _ptr(w_v), _ptr(scratch), nbytes, _stream(stream))

    def _check_proj(self, x, w_k, w_v) -> int:
        d = self.desc
        if x.dim() != 3 or tuple(x.shape[:2]) != (d.B, self.Lq):
            raise ValueError(f"x must be [{d.B}, {self.Lq}, hidden]")
        hidden = x.shape[2]
        for t in (x, w_k, w_v):
            if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
                raise ValueError("x, w_k, w_v must be contiguous CUDA bf16 tensors")
        for w in (w_k, w_v):
            if tuple(w.shape) != (d.H * 128, hidden):
                raise ValueError(f"weights must be [{d.H * 128}, {hidden}]")
        return hidden

    def attention(self, q: torch.Tensor, out: Optional[torch.Tensor] = None,
                  lse: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        self._check_io(q)
        if out is None:
            out = torch.empty_like(q)
        self._check_io(out)
        fn = L.chunk_attention_nvfp4kv if self.fp4 else L.chunk_attention_bf16kv
        fn(self.desc, self.cache, self.ring, _ptr(q), _ptr(out), _ptr(lse), _ptr(self.workspace),
           self.ws_bytes, _stream(stream))
        return out

    def step(self, q, k, v, out=None, lse=None, stream=None) -> torch.Tensor:
        """One AR step: evict when full, quantize-append, attend."""
        need = self.desc.C - min(self.free_frames(b) for b in range(self.desc.B))
        if need > 0:
            self.evict(need)
        self.append(k, v, stream)
        return self.attention(q, out, lse, stream)

    def _check_io(self, t: torch.Tensor) -> None:
        d = self.desc
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or tuple(
                t.shape) != (d.B, self.Lq, d.H, 128):
            raise ValueError(f"expected contiguous CUDA bf16 [{d.B}, {self.Lq}, {d.H}, 128], got "
                             f"{t.dtype} {tuple(t.shape)} on {t.device}")


def lse_merge(o_parts, lse_parts, q0: int = 0, q1: Optional[int] = None,
              out: Optional[torch.Tensor] = None, lse_out: Optional[torch.Tensor] = None,
              stream=None) -> torch.Tensor:
    """Attention over the union of disjoint key sets, from each set's result.

    o_parts: bf16 [B, Lq, H, 128] tensors (the shards' attention outputs),
    lse_parts: their f32 [B, H, Lq] lse.  Merges query rows [q0, q1) into
    out [B, q1 - q0, H, 128] (and lse_out [B, H, q1 - q0] if given)."""
    B, Lq, H, _ = o_parts[0].shape
    for t in o_parts:
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or tuple(
                t.shape) != (B, Lq, H, 128):
            raise ValueError("every part's out must be contiguous CUDA bf16 [B, Lq, H, 128]")
    for t in lse_parts:
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or tuple(
                t.shape) != (B, H, Lq):
            raise ValueError("every part's lse must be contiguous CUDA f32 [B, H, Lq]")
    q1 = Lq if q1 is None else q1
    if out is None:
        out = torch.empty((B, q1 - q0, H, 128), dtype=torch.bfloat16, device=o_parts[0].device)
    return lse_merge_ptrs([t.data_ptr() for t in o_parts], [t.data_ptr() for t in lse_parts],
                          B, Lq, H, q0, q1, out, lse_out, stream)


def lse_merge_ptrs(o_ptrs, lse_ptrs, B: int, Lq: int, H: int, q0: int, q1: int,
                   out: torch.Tensor, lse_out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """lse_merge with the parts given as device addresses (ints) of bf16
    [B, Lq, H, 128] outs and f32 [B, H, Lq] lses, e.g. other GPUs' buffers
    mapped into this process; out: bf16 [B, q1 - q0, H, 128]."""
    if tuple(out.shape) != (B, q1 - q0, H, 128) or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError(f"out must be contiguous bf16 [{B}, {q1 - q0}, {H}, 128]")
    if lse_out is not None and (tuple(lse_out.shape) != (B, H, q1 - q0) or
                                lse_out.dtype != torch.float32 or not lse_out.is_contiguous()):
        raise ValueError(f"lse_out must be contiguous f32 [{B}, {H}, {q1 - q0}]")
    L.nvkv_lse_merge(list(o_ptrs), list(lse_ptrs), B, H, Lq, q0, q1, _ptr(out), _ptr(lse_out),
                     _stream(stream))
    return out
