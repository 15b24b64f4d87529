"""nvfp4_kv_append_noalloc: the append for callers that cannot allocate
device memory (an engine plugin whose enqueue step may not allocate, or a
process whose device memory belongs to another allocator) keeps its amax
scratch in a fixed array inside the library instead of a caller plane.  Its
results must equal the regular nvfp4_kv_append's bit for bit, on two calls in
a row and again for a second stream whose first append reuses the array.

This file is named to be collected last, so that a run stopping at its first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import kvsynth

pytestmark = pytest.mark.gpu


def _pair(wl, shard=(0, 1)):
    import nvfp4_kv_cache_append_b200 as nv
    mk = lambda: nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, nv.NVKV_KV_NVFP4,
                            shard_rank=shard[0], shard_count=shard[1])
    return mk(), mk()


def _noalloc_append(nv, cache, k, v):
    c = cache.cache
    no_amax = nv._lib.nvkv_cache(c.k_data, c.v_data, c.k_scales, c.v_scales, None, c.s_g,
                                 c.status)
    nv._lib.nvfp4_kv_append_noalloc(cache.desc, no_amax, cache.ring, ctypes.c_void_p(k.data_ptr()),
                                    ctypes.c_void_p(v.data_ptr()),
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _same(a, b):
    for w in ("k", "v"):
        assert torch.equal(a.codes(w), b.codes(w))
        assert torch.equal(a.scales(w), b.scales(w))
    assert torch.equal(a.global_scales(), b.global_scales())
    assert bytes(a.ring) == bytes(b.ring)


@pytest.mark.parametrize("name", ["tiny", "stream5b"])
def test_noalloc_matches_regular_append(name):
    import nvfp4_kv_cache_append_b200 as nv
    wl = kvsynth.WORKLOADS[name]
    for stream_seed in (0, 7):          # second stream: first append reuses the array
        ref, new = _pair(wl)
        for step in (1, 2):             # two calls in a row (scale-fixing, then steady)
            x = kvsynth.chunk_qkv(wl, step, stream_seed)
            k, v = x["k"].cuda(), x["v"].cuda()
            ref.append(k, v)
            _noalloc_append(nv, new, k, v)
            torch.cuda.synchronize()
            _same(ref, new)
        assert int(new.amax.sum()) == 0     # the caller's amax plane was never used


def _two_appends(nv, wl, shard=(0, 1)):
    ref, new = _pair(wl, shard)
    for step in (1, 2):
        x = kvsynth.chunk_qkv(wl, step, 0)
        k, v = x["k"].cuda(), x["v"].cuda()
        ref.append(k, v)
        _noalloc_append(nv, new, k, v)
        torch.cuda.synchronize()
        _same(ref, new)
    assert int(new.amax.sum()) == 0


def test_noalloc_at_the_head_limit():
    """B * H = 256: the scratch array's last word is in use."""
    import nvfp4_kv_cache_append_b200 as nv
    wl = kvsynth.Workload(name="heads256", B=4, H=64, D=128, grid_h=4, grid_w=4, C=1, S=1, W=3, steps=2)
    _two_appends(nv, wl)


@pytest.mark.parametrize("rank", [0, 1])
def test_noalloc_shard(rank):
    """A shard of a two-way sequence-parallel KV split."""
    import nvfp4_kv_cache_append_b200 as nv
    _two_appends(nv, kvsynth.WORKLOADS["tiny"], shard=(rank, 2))


def test_noalloc_rejects_too_many_heads():
    import nvfp4_kv_cache_append_b200 as nv
    d = nv.nvkv_desc_init(8, 64, 4, 4, 1, 1, 3)          # 512 (b, h) pairs > 256
    r = nv.nvkv_ring_init(d)
    c = nv._lib.nvkv_cache(0x10000, 0x20000, 0x30000, 0x40000, None, 0x50000, 0x60000)
    with pytest.raises(nv.NvkvError) as e:
        nv._lib.nvfp4_kv_append_noalloc(d, c, r, ctypes.c_void_p(0x70000),
                                        ctypes.c_void_p(0x80000), None)
    assert e.value.status == nv._lib.STATUS_CODE["NVKV_ERR_UNSUPPORTED"]
    assert r.steps == 0
