"""C-ABI boundary on the CPU: the library loads, exports every declared entry
point, validates arguments before any launch, and its ring matches the
oracle's ring model.  No test here launches device work."""
import ctypes
import os
import random
import re

import pytest
import torch

import nvfp4_kv_cache_append_b200 as nv
from nvfp4_kv_cache_append_b200 import _lib as L
from oracle.ring import OracleRing

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_entry_points():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"^NVKV_API[^;(]*?\b([a-z_0-9]+)\s*\(", src, re.M)
    return names


def test_every_declared_symbol_is_exported():
    names = _declared_entry_points()
    assert len(names) >= 15
    raw = ctypes.CDLL(L.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n


def test_binding_covers_every_entry_point():
    for n in _declared_entry_points():
        assert n in L.lib.__dict__ or hasattr(L.lib, n)
        assert hasattr(L, n), f"no Python wrapper named {n}"


def test_struct_sizes_match_header_layout():
    assert ctypes.sizeof(L.nvkv_desc) == 4 * 17
    assert ctypes.sizeof(L.nvkv_cache) == 7 * 8
    assert ctypes.sizeof(L.nvkv_ring_stream) == 16 + 4 * 4 * 64
    assert ctypes.sizeof(L.nvkv_ring) == 32 + 16 * ctypes.sizeof(L.nvkv_ring_stream)


def _status(fn, *args):
    try:
        fn(*args)
    except L.NvkvError as e:
        return L.STATUS[e.status]
    return "NVKV_OK"


def test_desc_validation():
    ok = nv.nvkv_desc_init(1, 12, 30, 52, 3, 3, 18)
    assert ok.D == 128 and ok.rope_split[:] == [44, 42, 42] and ok.rope_base == 10000.0
    assert _status(nv.nvkv_desc_init, 17, 2, 8, 8, 1, 1, 3) == "NVKV_ERR_UNSUPPORTED"
    assert _status(nv.nvkv_desc_init, 1, 2, 8, 8, 4, 1, 3) == "NVKV_ERR_UNSUPPORTED"   # C > W
    assert _status(nv.nvkv_desc_init, 1, 2, 8, 8, 1, 40, 30) == "NVKV_ERR_UNSUPPORTED"
    assert _status(nv.nvkv_desc_init, 0, 2, 8, 8, 1, 1, 3) == "NVKV_ERR_INVALID_ARG"
    assert _status(nv.nvkv_desc_init, 1, 2, 8, 8, 1, 1, 3, 7) == "NVKV_ERR_INVALID_ARG"
    bad = nv.nvkv_desc_init(1, 2, 8, 8, 1, 1, 3)
    bad.D = 64
    assert L.lib.nvkv_ring_init(ctypes.byref(bad), ctypes.byref(L.nvkv_ring())) == 2
    bad.D = 128
    bad.magic = 0
    assert L.lib.nvkv_ring_init(ctypes.byref(bad), ctypes.byref(L.nvkv_ring())) == 5


def test_shard_validation():
    d = nv.nvkv_desc_init(1, 12, 30, 52, 3, 3, 18)
    assert (d.shard_rank, d.shard_count) == (0, 1)
    nv.nvkv_desc_set_shard(d, 3, 4)
    assert (d.shard_rank, d.shard_count) == (3, 4)
    for rank, count, want in [(2, 2, "NVKV_ERR_INVALID_ARG"), (0, 0, "NVKV_ERR_INVALID_ARG"),
                              (0, 17, "NVKV_ERR_INVALID_ARG"), (-1, 2, "NVKV_ERR_INVALID_ARG"),
                              (0, 7, "NVKV_ERR_INVALID_ARG")]:     # 1560 tokens do not split in 7
        e = nv.nvkv_desc_init(1, 12, 30, 52, 3, 3, 18)
        assert _status(nv.nvkv_desc_set_shard, e, rank, count) == want, (rank, count)
        assert (e.shard_rank, e.shard_count) == (0, 1)            # unchanged on error
    for kv in (nv.NVKV_KV_NVFP4, nv.NVKV_KV_BF16):
        t = nv.nvkv_desc_init(1, 12, 30, 52, 3, 3, 18, kv)
        nv.nvkv_desc_set_shard(t, 7, 8)                            # 195 tokens per shard (odd)
        # 195 tokens + one padding row per slot, 21 slots, 12 heads
        rows = 196 * 21 * 12
        assert L.nvkv_plane_bytes(t, L.NVKV_PLANE_K_DATA) == rows * (64 if kv == 0 else 256)
        if kv == nv.NVKV_KV_NVFP4:
            assert L.nvkv_plane_bytes(t, L.NVKV_PLANE_K_SCALES) == rows * 8 + 16
        nv.nvkv_desc_set_shard(t, 0, 1)
        assert (t.shard_rank, t.shard_count) == (0, 1)
        assert L.nvkv_plane_bytes(t, L.NVKV_PLANE_K_DATA) == 1560 * 21 * 12 * (64 if kv == 0 else 256)


def test_merge_validation_before_launch():
    fake = 1 << 20                                                 # never dereferenced
    for args, want in [((0, [], [], 1, 2, 8, 0, 8, fake), "NVKV_ERR_INVALID_ARG"),
                       ((17, [fake] * 17, [fake] * 17, 1, 2, 8, 0, 8, fake), "NVKV_ERR_INVALID_ARG"),
                       ((1, [fake], [fake], 1, 2, 8, 4, 4, fake), "NVKV_ERR_INVALID_ARG"),
                       ((1, [fake], [fake], 1, 2, 8, 0, 9, fake), "NVKV_ERR_INVALID_ARG"),
                       ((1, [0], [fake], 1, 2, 8, 0, 8, fake), "NVKV_ERR_INVALID_ARG"),
                       ((1, [fake + 8], [fake], 1, 2, 8, 0, 8, fake), "NVKV_ERR_ALIGNMENT"),
                       ((1, [fake], [fake + 2], 1, 2, 8, 0, 8, fake), "NVKV_ERR_ALIGNMENT"),
                       ((1, [fake], [fake], 1, 2, 8, 0, 8, fake + 4), "NVKV_ERR_ALIGNMENT")]:
        n, o, l = args[0], args[1], args[2]
        oa = (ctypes.c_void_p * max(n, 1))(*o)
        la = (ctypes.c_void_p * max(n, 1))(*l)
        st = L.lib.nvkv_lse_merge(n, oa, la, *args[3:], None, None)
        assert L.STATUS[st] == want, (args, L.STATUS[st])


def test_synced_merge_validation_before_launch():
    fake = 1 << 20                                                 # never dereferenced
    ok = dict(n=2, o=[fake, fake], l=[fake, fake], f=[fake, fake], rank=1, epoch=5, tmo=1000,
              status=fake)
    cases = [({}, None),
             ({"rank": 2}, "NVKV_ERR_INVALID_ARG"), ({"rank": -1}, "NVKV_ERR_INVALID_ARG"),
             ({"epoch": 0}, "NVKV_ERR_INVALID_ARG"), ({"tmo": 0}, "NVKV_ERR_INVALID_ARG"),
             ({"status": None}, "NVKV_ERR_INVALID_ARG"), ({"f": [fake, 0]}, "NVKV_ERR_INVALID_ARG"),
             ({"f": [fake, fake + 2]}, "NVKV_ERR_ALIGNMENT"), ({"status": fake + 1}, "NVKV_ERR_ALIGNMENT"),
             ({"o": [fake, fake + 8]}, "NVKV_ERR_ALIGNMENT"), ({"n": 0}, "NVKV_ERR_INVALID_ARG")]
    for change, want in cases:
        if want is None:
            continue                                               # a valid call would launch
        a = dict(ok, **change)
        n = a["n"]
        arr = lambda v: (ctypes.c_void_p * 2)(*v)
        st = L.lib.nvkv_lse_merge_synced(n, arr(a["o"]), arr(a["l"]), arr(a["f"]), a["rank"],
                                         a["epoch"], a["tmo"], a["status"], 1, 2, 8, 0, 8, fake,
                                         None, None)
        assert L.STATUS[st] == want, (change, L.STATUS[st])


def test_plane_bytes():
    d = nv.nvkv_desc_init(1, 12, 30, 52, 3, 3, 18)
    rows = 12 * 21 * 1560
    assert nv.nvkv_plane_bytes(d, L.NVKV_PLANE_K_DATA) == rows * 64
    assert nv.nvkv_plane_bytes(d, L.NVKV_PLANE_V_SCALES) == rows * 8 + 16
    assert nv.nvkv_plane_bytes(d, L.NVKV_PLANE_SCALE_G) == 2 * 12 * 4
    t = nv.nvkv_desc_init(1, 12, 30, 52, 3, 3, 18, nv.NVKV_KV_BF16)
    assert nv.nvkv_plane_bytes(t, L.NVKV_PLANE_K_DATA) == rows * 256
    assert nv.nvkv_plane_bytes(t, L.NVKV_PLANE_K_SCALES) == 0
    nv.nvkv_desc_set_shard(d, 1, 4)                        # a quarter of every frame
    assert nv.nvkv_plane_bytes(d, L.NVKV_PLANE_K_DATA) == rows // 4 * 64
    assert nv.nvkv_plane_bytes(d, L.NVKV_PLANE_V_SCALES) == rows // 4 * 8 + 16
    assert nv.nvkv_plane_bytes(d, L.NVKV_PLANE_SCALE_G) == 2 * 12 * 4


def _drive(desc, ring, sched_b, step):
    for b, sched in enumerate(sched_b):
        nv.kv_ring_begin_shot(desc, ring, b, sched[step])
    need = desc.C - min(desc.S + desc.W - ring.s[b].n_resident for b in range(desc.B))
    if need > 0:
        nv.kv_ring_evict(desc, ring, need)
    return nv.nvkv_ring_push_chunk(desc, ring)


@pytest.mark.parametrize("seed", range(6))
def test_ring_matches_oracle_model(seed):
    rnd = random.Random(seed)
    B, C, S = rnd.randint(1, 4), rnd.randint(1, 3), rnd.randint(0, 3)
    W = rnd.randint(2 * C, 9)        # room for a pinned per-shot sink plus one chunk
    desc = nv.nvkv_desc_init(B, 1, 2, 2, C, S, W)
    ring = nv.nvkv_ring_init(desc)
    steps = 40
    sched = []
    for b in range(B):
        ids, shot = [], 0
        for _ in range(steps):
            if rnd.random() < 0.15:
                shot += 1
            ids.append(shot)
        sched.append(ids)
    orings = [OracleRing(S, W, C) for _ in range(B)]
    for step in range(steps):
        slots = _drive(desc, ring, sched, step)
        for b in range(B):
            orings[b].begin_shot(sched[b][step])
            orings[b].step()
            sl, pos, frames, q0 = nv.nvkv_ring_visible(desc, ring, b)
            assert [list(x) for x in zip(frames, pos)] == [list(x) for x in orings[b].visible()]
            assert q0 == orings[b].query_pos0()
            st = ring.s[b]
            assert list(st.frame[:st.n_resident]) == orings[b].resident()
            used = list(st.slot[:st.n_resident])
            assert len(set(used)) == len(used) and all(0 <= p < S + W for p in used)
            assert set(slots[b]) <= set(used)


def test_evict_and_capacity_errors_leave_ring_unchanged():
    desc = nv.nvkv_desc_init(2, 1, 2, 2, 1, 1, 2)
    ring = nv.nvkv_ring_init(desc)
    for _ in range(3):
        nv.nvkv_ring_push_chunk(desc, ring)
    before = bytes(ring)
    assert _status(nv.nvkv_ring_push_chunk, desc, ring) == "NVKV_ERR_CAPACITY"
    assert _status(nv.kv_ring_evict, desc, ring, 3) == "NVKV_ERR_CAPACITY"
    assert _status(nv.kv_ring_evict, desc, ring, -1) == "NVKV_ERR_INVALID_ARG"
    assert bytes(ring) == before
    assert _status(nv.kv_ring_begin_shot, desc, ring, 2, 1) == "NVKV_ERR_INVALID_ARG"
    nv.kv_ring_begin_shot(desc, ring, 0, 2)
    assert _status(nv.kv_ring_begin_shot, desc, ring, 0, 1) == "NVKV_ERR_INVALID_ARG"
    other = nv.nvkv_desc_init(3, 1, 2, 2, 1, 1, 2)
    assert _status(nv.kv_ring_evict, other, ring, 1) == "NVKV_ERR_STATE"


def _fake_cache(base=0x10000):
    return L.nvkv_cache(base, base + 0x1000, base + 0x2000, base + 0x3000, base + 0x4000,
                        base + 0x5000, base + 0x6000)


def test_append_and_attention_validate_before_launch():
    d = nv.nvkv_desc_init(1, 2, 8, 8, 1, 1, 3)
    ring = nv.nvkv_ring_init(d)
    c = _fake_cache()
    kp, vp = ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000)
    assert _status(nv.nvfp4_kv_append, d, c, ring, None, vp) == "NVKV_ERR_INVALID_ARG"
    assert _status(nv.nvfp4_kv_append, d, c, ring, ctypes.c_void_p(0x20008), vp) == "NVKV_ERR_ALIGNMENT"
    assert _status(nv.bf16_kv_append, d, c, ring, kp, vp) == "NVKV_ERR_STATE"      # dtype
    bad = _fake_cache()
    bad.k_scales = 0x12008
    assert _status(nv.nvfp4_kv_append, d, bad, ring, kp, vp) == "NVKV_ERR_ALIGNMENT"
    qp, op = ctypes.c_void_p(0x40000), ctypes.c_void_p(0x50000)
    assert _status(nv.chunk_attention_nvfp4kv, d, c, ring, qp, op) == "NVKV_ERR_STATE"  # empty
    for _ in range(4):
        nv.nvkv_ring_push_chunk(d, ring)
    assert _status(nv.nvfp4_kv_append, d, c, ring, kp, vp) == "NVKV_ERR_CAPACITY"
    assert _status(L.nvfp4_kv_append_spatial_rope, d, c, ring, kp, vp) == "NVKV_ERR_CAPACITY"
    wide = nv.nvkv_desc_init(1, 2, 8, 91, 1, 1, 3)             # grid_w above 90
    assert _status(L.nvfp4_kv_append_spatial_rope, wide, c, nv.nvkv_ring_init(wide), kp,
                   vp) == "NVKV_ERR_UNSUPPORTED"
    fake = 1 << 20
    empty = nv.nvkv_ring_init(d)
    assert _status(L.nvkv_fp4qk_quantize_q, d, empty, kp, fake, fake, fake) == "NVKV_ERR_STATE"
    assert _status(L.nvkv_fp4qk_quantize_q, d, ring, None, fake, fake, fake) == "NVKV_ERR_INVALID_ARG"
    assert _status(L.nvkv_fp4qk_quantize_q, d, ring, kp, fake + 4, fake, fake) == "NVKV_ERR_ALIGNMENT"
    sc = L.nvkv_fp4qk_scores
    assert _status(sc, d, c, empty, fake, fake, fake, fake) == "NVKV_ERR_STATE"       # no append yet
    assert _status(sc, d, c, ring, None, fake, fake, fake) == "NVKV_ERR_INVALID_ARG"
    assert _status(sc, d, c, ring, fake + 8, fake, fake, fake) == "NVKV_ERR_ALIGNMENT"
    assert _status(sc, d, c, ring, fake, fake + 4, fake, fake) == "NVKV_ERR_ALIGNMENT"
    assert _status(sc, d, c, ring, fake, fake, fake, fake + 2) == "NVKV_ERR_ALIGNMENT"
    tw = nv.nvkv_desc_init(1, 2, 8, 8, 1, 1, 3, nv.NVKV_KV_BF16)
    rt = nv.nvkv_ring_init(tw)
    nv.nvkv_ring_push_chunk(tw, rt)
    assert _status(sc, tw, c, rt, fake, fake, fake, fake) == "NVKV_ERR_STATE"         # bf16 cache
    big = nv.nvkv_desc_init(1, 2, 50, 51, 1, 1, 3)               # grid_h + grid_w above 100
    rb = nv.nvkv_ring_init(big)
    nv.nvkv_ring_push_chunk(big, rb)
    assert _status(L.nvkv_fp4qk_quantize_q, big, rb, kp, fake, fake, fake) == "NVKV_ERR_UNSUPPORTED"
    sp = nv.nvkv_desc_init(1, 2, 8, 8, 1, 1, 3)
    sp.rope_split[0], sp.rope_split[1] = 40, 46
    assert _status(L.nvfp4_kv_append_spatial_rope, sp, c, nv.nvkv_ring_init(sp), kp,
                   vp) == "NVKV_ERR_UNSUPPORTED"
    assert _status(nv.chunk_attention_nvfp4kv, d, c, ring, None, op) == "NVKV_ERR_INVALID_ARG"
    assert _status(nv.chunk_attention_bf16kv, d, c, ring, qp, op) == "NVKV_ERR_STATE"
    split = nv.nvkv_desc_init(1, 2, 8, 8, 1, 1, 3)
    split.rope_split[0], split.rope_split[1] = 40, 46
    r2 = nv.nvkv_ring_init(split)
    nv.nvkv_ring_push_chunk(split, r2)
    assert _status(nv.chunk_attention_nvfp4kv, split, c, r2, qp, op) == "NVKV_ERR_UNSUPPORTED"


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_no_device_fails_loudly():
    d = nv.nvkv_desc_init(1, 2, 8, 8, 1, 1, 3)
    ring = nv.nvkv_ring_init(d)
    c = _fake_cache()
    st = _status(nv.nvfp4_kv_append, d, c, ring, ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000))
    assert st == "NVKV_ERR_CUDA"
    assert ring.steps == 0          # a failed launch does not advance the ring
    with pytest.raises(ValueError):
        nv.KVCache(1, 2, 8, 8, 1, 1, 3, device="cpu")


def test_status_strings():
    for code, name in L.STATUS.items():
        assert nv.nvkv_status_string(code)
    assert "unknown" in nv.nvkv_status_string(99)


def test_fault_hook_validation():
    assert _status(L.nvkv_debug_inject_fault, 9) == "NVKV_ERR_INVALID_ARG"
    assert _status(L.nvkv_debug_inject_fault, L.NVKV_FAULT_NONE) == "NVKV_OK"
