"""ctypes binding of libnvkv.so (include/nvkv.h): argument marshalling only.

Every function here has the name of the C entry point it calls.  Nothing in
this package computes any part of the path on the CPU; if the shared library
is missing or was built for another ABI version, importing the binding fails.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libnvkv.so")

NVKV_MAGIC = 0x4E564B56
NVKV_VERSION = 2
NVKV_HEAD_DIM = 128
NVKV_MAX_BATCH = 16
NVKV_MAX_FRAMES = 64
NVKV_MAX_CHUNK = 16
NVKV_MAX_SHARDS = 16
NVKV_KV_NVFP4 = 0
NVKV_KV_BF16 = 1
NVKV_FRAME_SINK = 1
NVKV_FRAME_PINNED = 2
NVKV_FRAME_SHOT_LAST = 4

(NVKV_PLANE_K_DATA, NVKV_PLANE_V_DATA, NVKV_PLANE_K_SCALES, NVKV_PLANE_V_SCALES,
 NVKV_PLANE_AMAX, NVKV_PLANE_SCALE_G, NVKV_PLANE_STATUS) = range(7)

STATUS = {0: "NVKV_OK", 1: "NVKV_ERR_INVALID_ARG", 2: "NVKV_ERR_UNSUPPORTED",
          3: "NVKV_ERR_ALIGNMENT", 4: "NVKV_ERR_CAPACITY", 5: "NVKV_ERR_STATE",
          6: "NVKV_ERR_CUDA", 7: "NVKV_ERR_TIMEOUT"}
STATUS_CODE = {v: k for k, v in STATUS.items()}


class nvkv_desc(ctypes.Structure):
    _fields_ = [("magic", ctypes.c_uint32), ("version", ctypes.c_uint32),
                ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("D", ctypes.c_int32),
                ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32), ("C", ctypes.c_int32),
                ("S", ctypes.c_int32), ("W", ctypes.c_int32), ("kv_dtype", ctypes.c_int32),
                ("rope_base", ctypes.c_float), ("rope_split", ctypes.c_int32 * 3),
                ("shard_rank", ctypes.c_int32), ("shard_count", ctypes.c_int32)]


class nvkv_cache(ctypes.Structure):
    _fields_ = [("k_data", ctypes.c_void_p), ("v_data", ctypes.c_void_p),
                ("k_scales", ctypes.c_void_p), ("v_scales", ctypes.c_void_p),
                ("amax", ctypes.c_void_p), ("s_g", ctypes.c_void_p),
                ("status", ctypes.c_void_p)]


class nvkv_ring_stream(ctypes.Structure):
    _fields_ = [("n_resident", ctypes.c_int32), ("shot", ctypes.c_int32),
                ("pin_next", ctypes.c_int32), ("n_appended", ctypes.c_int32),
                ("slot", ctypes.c_int32 * NVKV_MAX_FRAMES),
                ("frame", ctypes.c_int32 * NVKV_MAX_FRAMES),
                ("frame_shot", ctypes.c_int32 * NVKV_MAX_FRAMES),
                ("flags", ctypes.c_uint32 * NVKV_MAX_FRAMES)]


class nvkv_ring(ctypes.Structure):
    _fields_ = [("magic", ctypes.c_uint32), ("version", ctypes.c_uint32),
                ("B", ctypes.c_int32), ("capacity", ctypes.c_int32), ("C", ctypes.c_int32),
                ("S", ctypes.c_int32), ("scales_fixed", ctypes.c_int32),
                ("steps", ctypes.c_int32), ("s", nvkv_ring_stream * NVKV_MAX_BATCH)]


class NvkvError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({nvkv_status_string(status)})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libnvkv.so not built at {LIB_PATH}; run "
                          "`python nvfp4_kv_cache_append_b200/build.py` (needs nvcc)")
    L = ctypes.CDLL(LIB_PATH)
    D, C, R = ctypes.POINTER(nvkv_desc), ctypes.POINTER(nvkv_cache), ctypes.POINTER(nvkv_ring)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    i32p = ctypes.POINTER(ctypes.c_int32)
    sigs = {
        "nvkv_desc_init": (i32, [D, i32, i32, i32, i32, i32, i32, i32, i32]),
        "nvkv_desc_set_shard": (i32, [D, i32, i32]),
        "nvkv_kv_project": (i32, [D, vp, i32, vp, vp, vp, vp, vp, vp]),
        "nvkv_debug_inject_fault": (i32, [i32]),
        "nvfp4_kv_project_append": (i32, [D, C, R, vp, i32, vp, vp, vp, sz, vp]),
        "nvkv_lse_merge": (i32, [i32, ctypes.POINTER(vp), ctypes.POINTER(vp), i32, i32, i32, i32,
                                 i32, vp, vp, vp]),
        "nvkv_lse_merge_synced": (i32, [i32, ctypes.POINTER(vp), ctypes.POINTER(vp),
                                        ctypes.POINTER(vp), i32, ctypes.c_uint32,
                                        ctypes.c_uint32, vp, i32, i32, i32, i32, i32, vp, vp,
                                        vp]),
        "nvkv_plane_bytes": (sz, [D, i32]),
        "nvkv_ring_init": (i32, [D, R]),
        "kv_ring_evict": (i32, [D, R, i32]),
        "kv_ring_begin_shot": (i32, [D, R, i32, i32]),
        "nvkv_ring_visible": (i32, [D, R, i32, i32p, i32p, i32p, i32p]),
        "nvkv_ring_push_chunk": (i32, [D, R, i32p]),
        "nvfp4_kv_append": (i32, [D, C, R, vp, vp, vp]),
        "bf16_kv_append": (i32, [D, C, R, vp, vp, vp]),
        "nvfp4_kv_append_noalloc": (i32, [D, C, R, vp, vp, vp]),
        "nvfp4_kv_append_spatial_rope": (i32, [D, C, R, vp, vp, vp]),
        "nvkv_fp4qk_quantize_q": (i32, [D, R, vp, vp, vp, vp, vp]),
        "nvkv_fp4qk_scores": (i32, [D, C, R, vp, vp, vp, vp, vp]),
        "nvfp4_kv_overwrite": (i32, [D, C, R, vp, vp, vp]),
        "bf16_kv_overwrite": (i32, [D, C, R, vp, vp, vp]),
        "nvkv_attention_workspace_bytes": (sz, [D]),
        "chunk_attention_nvfp4kv": (i32, [D, C, R, vp, vp, vp, vp, sz, vp]),
        "chunk_attention_bf16kv": (i32, [D, C, R, vp, vp, vp, vp, sz, vp]),
        "nvkv_encode_e2m1": (i32, [vp, vp, sz, vp]),
        "nvkv_encode_block_scale": (i32, [vp, vp, sz, vp]),
        "nvkv_status_string": (ctypes.c_char_p, [i32]),
        "nvkv_version": (ctypes.c_uint32, []),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    if L.nvkv_version() != NVKV_VERSION:
        raise ImportError("libnvkv.so ABI version mismatch")
    return L


lib = _load()


def _check(status: int, what: str) -> None:
    if status != 0:
        raise NvkvError(status, what)


# ------------------------------------------------------------------ wrappers

def nvkv_status_string(status: int) -> str:
    return lib.nvkv_status_string(int(status)).decode()


def nvkv_desc_init(B, H, grid_h, grid_w, C, S, W, kv_dtype=NVKV_KV_NVFP4) -> nvkv_desc:
    d = nvkv_desc()
    _check(lib.nvkv_desc_init(ctypes.byref(d), B, H, grid_h, grid_w, C, S, W, kv_dtype),
           "nvkv_desc_init")
    return d


def nvkv_desc_set_shard(desc: nvkv_desc, rank: int, count: int) -> None:
    _check(lib.nvkv_desc_set_shard(ctypes.byref(desc), rank, count), "nvkv_desc_set_shard")


def nvkv_lse_merge(o_ptrs, lse_ptrs, B, H, Lq, q0, q1, out_ptr, lse_out_ptr=None, stream=0) -> None:
    """o_ptrs, lse_ptrs: sequences of device addresses (ints) of the parts."""
    n = len(o_ptrs)
    if len(lse_ptrs) != n:
        raise ValueError("one lse per part")
    oa = (ctypes.c_void_p * max(n, 1))(*o_ptrs)
    la = (ctypes.c_void_p * max(n, 1))(*lse_ptrs)
    _check(lib.nvkv_lse_merge(n, oa, la, B, H, Lq, q0, q1, out_ptr, lse_out_ptr, stream),
           "nvkv_lse_merge")


def nvkv_lse_merge_synced(o_ptrs, lse_ptrs, flag_ptrs, rank, epoch, timeout_us, status_ptr, B, H,
                          Lq, q0, q1, out_ptr, lse_out_ptr=None, stream=0) -> None:
    """nvkv_lse_merge behind the bounded cross-rank flag barrier; flag_ptrs:
    device addresses (ints) of every rank's signal array."""
    n = len(o_ptrs)
    if len(lse_ptrs) != n or len(flag_ptrs) != n:
        raise ValueError("one lse and one flag array per part")
    oa = (ctypes.c_void_p * max(n, 1))(*o_ptrs)
    la = (ctypes.c_void_p * max(n, 1))(*lse_ptrs)
    fa = (ctypes.c_void_p * max(n, 1))(*flag_ptrs)
    _check(lib.nvkv_lse_merge_synced(n, oa, la, fa, rank, epoch, timeout_us, status_ptr, B, H, Lq,
                                     q0, q1, out_ptr, lse_out_ptr, stream),
           "nvkv_lse_merge_synced")


NVKV_FAULT_NONE = 0
NVKV_FAULT_SKIP_FIRST_STAGE = 1


def nvkv_debug_inject_fault(fault: int) -> None:
    _check(lib.nvkv_debug_inject_fault(fault), "nvkv_debug_inject_fault")


def nvkv_kv_project(desc, x_ptr, hidden, wk_ptr, wv_ptr, k_out_ptr, v_out_ptr, status_ptr,
                    stream=0) -> None:
    _check(lib.nvkv_kv_project(ctypes.byref(desc), x_ptr, hidden, wk_ptr, wv_ptr, k_out_ptr,
                               v_out_ptr, status_ptr, stream), "nvkv_kv_project")


def nvfp4_kv_project_append(desc, cache, ring, x_ptr, hidden, wk_ptr, wv_ptr, scratch_ptr,
                            scratch_bytes, stream=0) -> None:
    _check(lib.nvfp4_kv_project_append(ctypes.byref(desc), ctypes.byref(cache), ctypes.byref(ring),
                                       x_ptr, hidden, wk_ptr, wv_ptr, scratch_ptr, scratch_bytes,
                                       stream), "nvfp4_kv_project_append")


def nvkv_plane_bytes(desc: nvkv_desc, plane: int) -> int:
    return int(lib.nvkv_plane_bytes(ctypes.byref(desc), plane))


def nvkv_ring_init(desc: nvkv_desc) -> nvkv_ring:
    r = nvkv_ring()
    _check(lib.nvkv_ring_init(ctypes.byref(desc), ctypes.byref(r)), "nvkv_ring_init")
    return r


def kv_ring_evict(desc: nvkv_desc, ring: nvkv_ring, n_frames: int) -> None:
    _check(lib.kv_ring_evict(ctypes.byref(desc), ctypes.byref(ring), n_frames), "kv_ring_evict")


def kv_ring_begin_shot(desc: nvkv_desc, ring: nvkv_ring, b: int, shot_id: int) -> None:
    _check(lib.kv_ring_begin_shot(ctypes.byref(desc), ctypes.byref(ring), b, shot_id),
           "kv_ring_begin_shot")


def nvkv_ring_visible(desc: nvkv_desc, ring: nvkv_ring, b: int):
    """(slots, rope_pos, frames, query_pos0) of what stream b's newest chunk sees."""
    n_max = NVKV_MAX_FRAMES
    slots, pos, frames = (ctypes.c_int32 * n_max)(), (ctypes.c_int32 * n_max)(), (ctypes.c_int32 * n_max)()
    q0 = ctypes.c_int32()
    n = lib.nvkv_ring_visible(ctypes.byref(desc), ctypes.byref(ring), b, slots, pos, frames,
                              ctypes.byref(q0))
    if n < 0:
        raise NvkvError(STATUS_CODE["NVKV_ERR_INVALID_ARG"], "nvkv_ring_visible")
    return list(slots[:n]), list(pos[:n]), list(frames[:n]), q0.value


def nvkv_ring_push_chunk(desc: nvkv_desc, ring: nvkv_ring):
    """Host-only ring update of one append; returns the slots [B][C]."""
    out = (ctypes.c_int32 * (NVKV_MAX_BATCH * NVKV_MAX_CHUNK))()
    _check(lib.nvkv_ring_push_chunk(ctypes.byref(desc), ctypes.byref(ring), out),
           "nvkv_ring_push_chunk")
    return [list(out[b * desc.C:(b + 1) * desc.C]) for b in range(desc.B)]


def nvfp4_kv_append(desc, cache, ring, k_ptr, v_ptr, stream=0) -> None:
    _check(lib.nvfp4_kv_append(ctypes.byref(desc), ctypes.byref(cache), ctypes.byref(ring),
                               k_ptr, v_ptr, stream), "nvfp4_kv_append")


def nvfp4_kv_overwrite(desc, cache, ring, k_ptr, v_ptr, stream=0) -> None:
    _check(lib.nvfp4_kv_overwrite(ctypes.byref(desc), ctypes.byref(cache), ctypes.byref(ring),
                                  k_ptr, v_ptr, stream), "nvfp4_kv_overwrite")


def bf16_kv_overwrite(desc, cache, ring, k_ptr, v_ptr, stream=0) -> None:
    _check(lib.bf16_kv_overwrite(ctypes.byref(desc), ctypes.byref(cache), ctypes.byref(ring),
                                 k_ptr, v_ptr, stream), "bf16_kv_overwrite")


def nvfp4_kv_append_noalloc(desc, cache, ring, k_ptr, v_ptr, stream=0) -> None:
    _check(lib.nvfp4_kv_append_noalloc(ctypes.byref(desc), ctypes.byref(cache),
                                       ctypes.byref(ring), k_ptr, v_ptr, stream),
           "nvfp4_kv_append_noalloc")


def nvfp4_kv_append_spatial_rope(desc, cache, ring, k_ptr, v_ptr, stream=0) -> None:
    _check(lib.nvfp4_kv_append_spatial_rope(ctypes.byref(desc), ctypes.byref(cache),
                                            ctypes.byref(ring), k_ptr, v_ptr, stream),
           "nvfp4_kv_append_spatial_rope")


def nvkv_fp4qk_quantize_q(desc, ring, q_ptr, codes_ptr, scales_ptr, s_gq_ptr, stream=0) -> None:
    _check(lib.nvkv_fp4qk_quantize_q(ctypes.byref(desc), ctypes.byref(ring), q_ptr, codes_ptr,
                                     scales_ptr, s_gq_ptr, stream), "nvkv_fp4qk_quantize_q")


def nvkv_fp4qk_scores(desc, cache, ring, q_codes_ptr, q_scales_ptr, s_gq_ptr, out_ptr,
                      stream=0) -> None:
    _check(lib.nvkv_fp4qk_scores(ctypes.byref(desc), ctypes.byref(cache), ctypes.byref(ring),
                                 q_codes_ptr, q_scales_ptr, s_gq_ptr, out_ptr, stream),
           "nvkv_fp4qk_scores")


def bf16_kv_append(desc, cache, ring, k_ptr, v_ptr, stream=0) -> None:
    _check(lib.bf16_kv_append(ctypes.byref(desc), ctypes.byref(cache), ctypes.byref(ring),
                              k_ptr, v_ptr, stream), "bf16_kv_append")


def nvkv_attention_workspace_bytes(desc) -> int:
    return int(lib.nvkv_attention_workspace_bytes(ctypes.byref(desc)))


def chunk_attention_nvfp4kv(desc, cache, ring, q_ptr, out_ptr, lse_ptr=None, ws_ptr=None,
                            ws_bytes=0, stream=0) -> None:
    _check(lib.chunk_attention_nvfp4kv(ctypes.byref(desc), ctypes.byref(cache),
                                       ctypes.byref(ring), q_ptr, out_ptr, lse_ptr, ws_ptr,
                                       ws_bytes, stream), "chunk_attention_nvfp4kv")


def chunk_attention_bf16kv(desc, cache, ring, q_ptr, out_ptr, lse_ptr=None, ws_ptr=None,
                           ws_bytes=0, stream=0) -> None:
    _check(lib.chunk_attention_bf16kv(ctypes.byref(desc), ctypes.byref(cache),
                                      ctypes.byref(ring), q_ptr, out_ptr, lse_ptr, ws_ptr,
                                      ws_bytes, stream), "chunk_attention_bf16kv")


def nvkv_encode_e2m1(y_ptr, codes_ptr, n, stream=0) -> None:
    _check(lib.nvkv_encode_e2m1(y_ptr, codes_ptr, n, stream), "nvkv_encode_e2m1")


def nvkv_encode_block_scale(t_ptr, codes_ptr, n, stream=0) -> None:
    _check(lib.nvkv_encode_block_scale(t_ptr, codes_ptr, n, stream), "nvkv_encode_block_scale")


def nvkv_version() -> int:
    return int(lib.nvkv_version())
