"""CPU oracle for the NVFP4 KV-cache append and chunk attention path.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg import this package; the product path never does.  It shares no
code with the CUDA library (``nvfp4_kv_cache_append_b200``) and never imports
it; the only common module is ``kvsynth`` (seeded inputs, no arithmetic).

The arithmetic lives in ``nvfp4_oracle.c`` (plain C: FP32 scale arithmetic as
the format fixes it, fp64 for everything after dequantization).  This module
builds it with gcc, loads it with ctypes and wraps it for numpy arrays.
Every function names the passage it follows in the C source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

ROPE_SPLIT = (44, 42, 42)
ROPE_BASE = 10000.0


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP, no fast-math, no FP contraction)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                               "-ffp-contract=off", "-fno-fast-math", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
            f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
            f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
            i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
            i64p = np.ctypeslib.ndpointer(np.int64, flags="C_CONTIGUOUS")
            L.oracle_e2m1_decode.restype = ctypes.c_double
            L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
            L.oracle_e4m3_decode.restype = ctypes.c_double
            L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
            L.oracle_e2m1_encode.restype = ctypes.c_uint8
            L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
            L.oracle_e4m3_encode.restype = ctypes.c_uint8
            L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
            L.oracle_global_scale.restype = ctypes.c_float
            L.oracle_global_scale.argtypes = [ctypes.c_float]
            L.oracle_amax.restype = ctypes.c_float
            L.oracle_amax.argtypes = [f32p, ctypes.c_int64]
            L.oracle_quantize_block16.restype = None
            L.oracle_quantize_block16.argtypes = [f32p, ctypes.c_float, u8p, u8p]
            L.oracle_quantize_rows.restype = None
            L.oracle_quantize_rows.argtypes = [f32p, ctypes.c_int64, ctypes.c_float, u8p, u8p]
            L.oracle_dequant_rows.restype = None
            L.oracle_dequant_rows.argtypes = [u8p, u8p, ctypes.c_int64, ctypes.c_float, f64p]
            L.oracle_rope3d.restype = None
            L.oracle_rope3d.argtypes = [f64p, i32p, i32p, ctypes.c_double]
            L.oracle_attention_rows.restype = None
            L.oracle_attention_rows.argtypes = [f32p, f64p, f64p, ctypes.c_int64, i32p, i32p, i32p,
                                                i32p, i64p, ctypes.c_int64, ctypes.c_int, i32p,
                                                ctypes.c_double, f64p, f64p]
            fp = ctypes.POINTER(ctypes.c_float)
            L.oracle_rope_cs_f32.restype = None
            L.oracle_rope_cs_f32.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_double, fp, fp]
            L.oracle_rope3d_f32.restype = None
            L.oracle_rope3d_f32.argtypes = [f32p, i32p, i32p, ctypes.c_double]
            L.oracle_k_spatial_rope_f32.restype = None
            L.oracle_k_spatial_rope_f32.argtypes = [f32p, ctypes.c_int64, i32p, ctypes.c_int, i32p,
                                                    ctypes.c_double]
            L.oracle_q_row_global_scale.restype = ctypes.c_float
            L.oracle_q_row_global_scale.argtypes = [f32p]
            L.oracle_q_for_frame.restype = None
            L.oracle_q_for_frame.argtypes = [f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, i32p,
                                             ctypes.c_double, ctypes.c_float, u8p, u8p]
            L.oracle_fp4_dot.restype = ctypes.c_double
            L.oracle_fp4_dot.argtypes = [u8p, u8p, ctypes.c_float, u8p, u8p, ctypes.c_float]
            L.oracle_attention_rows_fp4qk.restype = None
            L.oracle_attention_rows_fp4qk.argtypes = [f32p, f64p, f64p, ctypes.c_int64, i32p,
                                                      i32p, i32p, i64p, ctypes.c_int64,
                                                      ctypes.c_int, i32p, ctypes.c_double,
                                                      ctypes.c_int, f64p, f64p]
            L.oracle_block_scale_code.restype = ctypes.c_uint8
            L.oracle_block_scale_code.argtypes = [ctypes.c_float]
            L.oracle_e2m1_encode_array.restype = None
            L.oracle_e2m1_encode_array.argtypes = [f32p, ctypes.c_int64, u8p]
            L.oracle_block_scale_code_array.restype = None
            L.oracle_block_scale_code_array.argtypes = [f32p, ctypes.c_int64, u8p]
            _lib = L
    return _lib


# ------------------------------------------------------------------ scalars

def e2m1_decode(code: int) -> float:
    return lib().oracle_e2m1_decode(int(code))


def e4m3_decode(code: int) -> float:
    return lib().oracle_e4m3_decode(int(code))


def e2m1_encode(y: float) -> int:
    return int(lib().oracle_e2m1_encode(float(y)))


def e4m3_encode(t: float) -> int:
    return int(lib().oracle_e4m3_encode(float(t)))


def block_scale_code(t: float) -> int:
    """E4M3 code of a block-scale ratio t (clamped at 448)."""
    return int(lib().oracle_block_scale_code(float(t)))


def e2m1_encode_array(y: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(y, np.float32).reshape(-1)
    out = np.empty(a.size, np.uint8)
    lib().oracle_e2m1_encode_array(a, a.size, out)
    return out.reshape(np.shape(y))


def block_scale_code_array(t: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(t, np.float32).reshape(-1)
    out = np.empty(a.size, np.uint8)
    lib().oracle_block_scale_code_array(a, a.size, out)
    return out.reshape(np.shape(t))


def global_scale(amax: float) -> float:
    return float(lib().oracle_global_scale(float(np.float32(amax))))


# ------------------------------------------------------------------- arrays

def _as_f32(x) -> np.ndarray:
    """bf16/float tensors or arrays -> contiguous float32 numpy (exact for bf16)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu").float().numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def amax(x) -> float:
    a = _as_f32(x).reshape(-1)
    return float(lib().oracle_amax(a, a.size))


def quantize_block16(x, s_g: float):
    a = _as_f32(x).reshape(16)
    codes = np.zeros(8, np.uint8)
    scale = np.zeros(1, np.uint8)
    lib().oracle_quantize_block16(a, float(np.float32(s_g)), codes, scale)
    return codes, int(scale[0])


def quantize_rows(x, s_g: float):
    """x [..., 128] -> (codes [..., 64] u8, scales [..., 8] u8) with one global scale."""
    a = _as_f32(x)
    lead = a.shape[:-1]
    assert a.shape[-1] == 128
    a = a.reshape(-1, 128)
    n = a.shape[0]
    codes = np.zeros((n, 64), np.uint8)
    scales = np.zeros((n, 8), np.uint8)
    if n:
        lib().oracle_quantize_rows(a, n, float(np.float32(s_g)), codes, scales)
    return codes.reshape(*lead, 64), scales.reshape(*lead, 8)


def dequant_rows(codes: np.ndarray, scales: np.ndarray, s_g: float) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    lead = c.shape[:-1]
    c2 = c.reshape(-1, 64)
    s2 = s.reshape(-1, 8)
    out = np.zeros((c2.shape[0], 128), np.float64)
    if c2.shape[0]:
        lib().oracle_dequant_rows(c2, s2, c2.shape[0], float(np.float32(s_g)), out)
    return out.reshape(*lead, 128)


def rope3d(x, pos3, split=ROPE_SPLIT, base=ROPE_BASE) -> np.ndarray:
    """Rotate one 128-vector (fp64) at 3D position (frame, h, w)."""
    v = np.array(x, dtype=np.float64).reshape(128).copy()
    lib().oracle_rope3d(v, np.asarray(pos3, np.int32), np.asarray(split, np.int32), float(base))
    return v


def attention_rows(q, k: np.ndarray, v: np.ndarray, k_frame_pos, k_tok, q_frame_pos, q_tok,
                   rows, grid_w: int, split=ROPE_SPLIT, base=ROPE_BASE):
    """Chunk attention for one (batch, head) on the listed query rows (fp64).

    q [Lq, 128] (pre-RoPE bf16 values), k/v [Lk, 128] fp64 dequantized,
    position arrays as in ``oracle_attention_rows``.  Returns (out [n, 128], lse [n]).
    """
    qa = _as_f32(q).reshape(-1, 128)
    ka = np.ascontiguousarray(k, np.float64).reshape(-1, 128)
    va = np.ascontiguousarray(v, np.float64).reshape(-1, 128)
    Lk = ka.shape[0]
    rows = np.ascontiguousarray(rows, np.int64)
    out = np.zeros((rows.size, 128), np.float64)
    lse = np.zeros(rows.size, np.float64)
    lib().oracle_attention_rows(qa, ka, va, Lk, np.ascontiguousarray(k_frame_pos, np.int32),
                                np.ascontiguousarray(k_tok, np.int32),
                                np.ascontiguousarray(q_frame_pos, np.int32),
                                np.ascontiguousarray(q_tok, np.int32), rows, rows.size, int(grid_w),
                                np.asarray(split, np.int32), float(base), out, lse)
    return out, lse


# ------------------------------------------ block-scaled FP4 Q K^T (a reading)
# The steps and their precision are stated in nvfp4_oracle.c, section
# "block-scaled FP4 Q K^T (a reading)".

def rope_cs_f32(pos: int, i: int, d: int, base: float = ROPE_BASE):
    """cos and sin of pair i of a width-d segment at position pos, each rounded to float."""
    c, s = ctypes.c_float(), ctypes.c_float()
    lib().oracle_rope_cs_f32(int(pos), int(i), int(d), float(base), ctypes.byref(c), ctypes.byref(s))
    return np.float32(c.value), np.float32(s.value)


def rope3d_f32(x, pos3, split=ROPE_SPLIT, base=ROPE_BASE) -> np.ndarray:
    """One 128-vector rotated in float (the quantizer-feeding rotation)."""
    v = _as_f32(x).reshape(128).copy()
    lib().oracle_rope3d_f32(v, np.asarray(pos3, np.int32), np.asarray(split, np.int32), float(base))
    return v


def k_spatial_rope_f32(k, tok, grid_w: int, split=ROPE_SPLIT, base=ROPE_BASE) -> np.ndarray:
    """K rows [n, 128] with their h and w segments rotated at each row's token."""
    a = _as_f32(k).reshape(-1, 128).copy()
    t = np.ascontiguousarray(tok, np.int32).reshape(-1)
    assert t.size == a.shape[0]
    if a.shape[0]:
        lib().oracle_k_spatial_rope_f32(a, a.shape[0], t, int(grid_w), np.asarray(split, np.int32),
                                        float(base))
    return a


def q_row_global_scale(q) -> float:
    a = _as_f32(q).reshape(128)
    return float(lib().oracle_q_row_global_scale(a))


def q_for_frame(q, dpos: int, q_tok: int, grid_w: int, s_gq: float, split=ROPE_SPLIT,
                base=ROPE_BASE):
    """Q_fk of one row for relative frame index dpos: (codes [64], scales [8])."""
    a = _as_f32(q).reshape(128)
    codes = np.zeros(64, np.uint8)
    scales = np.zeros(8, np.uint8)
    lib().oracle_q_for_frame(a, int(dpos), int(q_tok), int(grid_w), np.asarray(split, np.int32),
                             float(base), float(np.float32(s_gq)), codes, scales)
    return codes, scales


def fp4_dot(ca, sa, ga: float, cb, sb, gb: float) -> float:
    """Block form of one FP4 x FP4 dot product (integer code sums x block scales)."""
    f = lambda x: np.ascontiguousarray(x, np.uint8)
    return float(lib().oracle_fp4_dot(f(ca), f(sa), float(np.float32(ga)), f(cb), f(sb),
                                      float(np.float32(gb))))


def attention_rows_fp4qk(q, k: np.ndarray, v: np.ndarray, k_frame_pos, q_frame_pos, q_tok, rows,
                         grid_w: int, quantize_q: bool = True, split=ROPE_SPLIT, base=ROPE_BASE):
    """Chunk attention of one (batch, head) with FP4 logits: q [Lq, 128]
    pre-RoPE, k [Lk, 128] the cached K' rows dequantized (spatially rotated
    keys, quantized), v [Lk, 128] fp64.  ``quantize_q=False`` keeps Q_fk in
    float.  Returns (out [n, 128], lse [n])."""
    qa = _as_f32(q).reshape(-1, 128)
    ka = np.ascontiguousarray(k, np.float64).reshape(-1, 128)
    va = np.ascontiguousarray(v, np.float64).reshape(-1, 128)
    Lk = ka.shape[0]
    rows = np.ascontiguousarray(rows, np.int64)
    out = np.zeros((rows.size, 128), np.float64)
    lse = np.zeros(rows.size, np.float64)
    lib().oracle_attention_rows_fp4qk(qa, ka, va, Lk, np.ascontiguousarray(k_frame_pos, np.int32),
                                      np.ascontiguousarray(q_frame_pos, np.int32),
                                      np.ascontiguousarray(q_tok, np.int32), rows, rows.size,
                                      int(grid_w), np.asarray(split, np.int32), float(base),
                                      1 if quantize_q else 0, out, lse)
    return out, lse
