"""Quantize-append parity: every code and scale byte the CUDA path writes
equals the oracle's, at every step, in the physical slot the ring assigned;
nothing outside those slots is touched."""
import numpy as np
import pytest
import torch

import kvsynth
import oracle
from oracle.stream import OracleStream
from tests._harness import LibStream, to_gpu

pytestmark = pytest.mark.gpu


def _check_new_frames(lib: LibStream, ora: OracleStream, new):
    wl = lib.wl
    for b, fids in new.items():
        for fid in fids:
            rows = lib.frame_rows(b, fid)
            e = ora.frame(b, fid)
            for w in ("k", "v"):
                got_c = lib.cache.codes(w)[b, :, rows].cpu().numpy()
                got_s = lib.cache.scales(w)[b, :, rows].cpu().numpy()
                assert np.array_equal(got_c, e[w + "_codes"]), (b, fid, w)
                assert np.array_equal(got_s, e[w + "_scales"]), (b, fid, w)


@pytest.mark.parametrize("name", ["tiny", "stream1p3b", "stream5b"])
def test_append_bit_exact(name):
    import nvfp4_kv_cache_append_b200 as nv
    wl = kvsynth.WORKLOADS[name]
    lib = LibStream(wl, nv.NVKV_KV_NVFP4)
    ora = OracleStream(wl, seed=0, keep_inputs=False)
    for step in range(1, wl.steps + 1):
        x = kvsynth.chunk_qkv(wl, step, 0)
        new = ora.step(k=x["k"], v=x["v"], q=x["q"])
        g = to_gpu(x)
        lib.step(g["q"], g["k"], g["v"])
        torch.cuda.synchronize()
        if step == 1:
            assert np.array_equal(lib.cache.global_scales().cpu().numpy(), ora.s_g)
        _check_new_frames(lib, ora, new)
    assert lib.cache.device_status() == 0
    # after the ring wrapped, every resident frame still matches
    for b in range(wl.B):
        for fid in ora.rings[b].resident():
            _check_new_frames(lib, ora, {b: [fid]})


def test_append_multishot_bit_exact():
    import nvfp4_kv_cache_append_b200 as nv
    wl = kvsynth.WORKLOADS["multishot"]
    sched = kvsynth.shot_schedule(wl, 0)
    lib = LibStream(wl, nv.NVKV_KV_NVFP4, sched=sched)
    ora = OracleStream(wl, seed=0, shot_sched=sched, keep_inputs=False)
    for step in range(1, wl.steps + 1):
        x = kvsynth.chunk_qkv(wl, step, 0)
        new = ora.step(k=x["k"], v=x["v"], q=x["q"])
        g = to_gpu(x)
        lib.step(g["q"], g["k"], g["v"], with_lse=False)
        torch.cuda.synchronize()
        if step in (1, 2, 9, 16, 17, 24):
            _check_new_frames(lib, ora, new)
        for b in range(wl.B):
            assert lib.cache.visible(b)[2] == [f for f, _ in ora.rings[b].visible()]


def test_append_leaves_other_bytes_alone():
    import nvfp4_kv_cache_append_b200 as nv
    wl = kvsynth.WORKLOADS["tiny"]
    lib = LibStream(wl, nv.NVKV_KV_NVFP4)
    for t in (lib.cache.k_data, lib.cache.v_data, lib.cache.k_scales, lib.cache.v_scales):
        t.fill_(0xA5)
    x = to_gpu(kvsynth.chunk_qkv(wl, 1, 0))
    lib.step(x["q"], x["k"], x["v"])
    torch.cuda.synchronize()
    rows = lib.frame_rows(0, 0)
    for w in ("k", "v"):
        c = lib.cache.codes(w)[0].clone()
        s = lib.cache.scales(w)[0].clone()
        c[:, rows] = 0xA5
        s[:, rows] = 0xA5
        assert bool((c == 0xA5).all()) and bool((s == 0xA5).all())
    pad = lib.cache.k_scales[-16:]
    assert bool((pad == 0xA5).all())


def test_zero_first_chunk_gives_unit_scale_and_zero_codes():
    import nvfp4_kv_cache_append_b200 as nv
    wl = kvsynth.WORKLOADS["tiny"]
    lib = LibStream(wl, nv.NVKV_KV_NVFP4)
    z = torch.zeros(wl.B, wl.Lq, wl.H, 128, dtype=torch.bfloat16, device="cuda")
    lib.step(z, z, z)
    torch.cuda.synchronize()
    assert bool((lib.cache.global_scales() == 1.0).all())
    rows = lib.frame_rows(0, 0)
    assert int(lib.cache.codes("k")[0, :, rows].sum()) == 0
    assert int(lib.cache.scales("v")[0, :, rows].sum()) == 0


def test_bf16_twin_append_copies_exactly():
    import nvfp4_kv_cache_append_b200 as nv
    wl = kvsynth.WORKLOADS["stream5b"]
    lib = LibStream(wl, nv.NVKV_KV_BF16)
    for step in range(1, wl.steps + 1):
        x = kvsynth.chunk_qkv(wl, step, 0)
        g = to_gpu(x)
        lib.step(g["q"], g["k"], g["v"], with_lse=False)
        torch.cuda.synchronize()
        for c in range(wl.C):
            fid = (step - 1) * wl.C + c
            rows = lib.frame_rows(0, fid)
            for w in ("k", "v"):
                want = x[w][0, c * wl.T:(c + 1) * wl.T].transpose(0, 1)
                got = lib.cache.codes(w)[0, :, rows].cpu()
                assert torch.equal(got.view(torch.int16), want.contiguous().view(torch.int16))


@pytest.mark.parametrize("first_scale,later_scale", [
    (2.0 ** -100, 2.0 ** -100),   # tiny global scale: divisor below 2^-64 (IEEE-division blocks)
    (2.0 ** -60, 1.0),            # later chunks far above the first: saturated codes
    (1.0, 2.0 ** 40),             # block scales clamped at 448, quotients up to ~2^40
    (1.0, 2.0 ** 70),             # quotients beyond 2^64 (IEEE-division blocks)
    (2.0 ** 60, 2.0 ** 60),       # divisors near 2^64
])
def test_append_extreme_scales_bit_exact(first_scale, later_scale):
    """Codes and scales stay bit-exact when the scales leave the usual range:
    both the shared-reciprocal division and the IEEE-division fallback of the
    append kernel meet the oracle's fl32(x / (s_b s_g))."""
    import nvfp4_kv_cache_append_b200 as nv
    wl = kvsynth.WORKLOADS["tiny"]
    lib = LibStream(wl, nv.NVKV_KV_NVFP4)
    ora = OracleStream(wl, seed=0, keep_inputs=False)
    for step in range(1, 5):
        x = kvsynth.chunk_qkv(wl, step, 0)
        sc = first_scale if step == 1 else later_scale
        k = (x["k"].float() * sc).to(torch.bfloat16)
        v = (x["v"].float() * sc).to(torch.bfloat16)
        new = ora.step(k=k, v=v, q=x["q"])
        lib.cache.append(k.cuda(), v.cuda())
        torch.cuda.synchronize()
        if step == 1:
            assert np.array_equal(lib.cache.global_scales().cpu().numpy(), ora.s_g)
        _check_new_frames(lib, ora, new)
    assert lib.cache.device_status() == 0


ODD60 = kvsynth.Workload("odd60", B=2, H=3, D=128, grid_h=6, grid_w=10, C=2, S=1, W=6, steps=5)


@pytest.mark.parametrize("name,count,steps", [("tiny", 1, 6), ("tiny", 4, 6), ("odd60", 4, 5),
                                              ("stream1p3b", 1, 2), ("stream5b", 2, 2)])
def test_spatial_rope_append_bit_exact(name, count, steps):
    """The append of the block-scaled FP4 Q K^T reading (K's h and w pairs
    rotated in float before quantizing) against the oracle's fp4_qk stream:
    s_g and every new frame's codes and scales bit for bit, on whole caches
    and shards (odd ones included) across ring wrap."""
    import nvfp4_kv_cache_append_b200 as nv
    from oracle.merge import shard_tokens
    wl = ODD60 if name == "odd60" else kvsynth.WORKLOADS[name]
    shards = [nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, nv.NVKV_KV_NVFP4,
                         shard_rank=r, shard_count=count) for r in range(count)]
    ora = OracleStream(wl, seed=7, keep_inputs=False, fp4_qk=True)
    for step in range(1, steps + 1):
        x = kvsynth.chunk_qkv(wl, step, 7)
        new = ora.step(k=x["k"], v=x["v"], q=x["q"])
        g = to_gpu(x)
        for c in shards:
            need = wl.C - min(c.free_frames(b) for b in range(wl.B))
            if need > 0:
                c.evict(need)
            c.append_spatial_rope(g["k"], g["v"])
        torch.cuda.synchronize()
        for r, c in enumerate(shards):
            assert c.device_status() == 0
            assert np.array_equal(c.global_scales().cpu().numpy(), ora.s_g), (step, r)
            t0, t1 = shard_tokens(wl.T, count, r)
            ts, tr = c.Ts, c.Tr
            for b in range(wl.B):
                st = c.ring.s[b]
                slot_of = {st.frame[i]: st.slot[i] for i in range(st.n_resident)}
                for fid in new[b]:
                    p = slot_of[fid]
                    e = ora.frame(b, fid)
                    rows = slice(p * tr, p * tr + ts)
                    for w in ("k", "v"):
                        assert np.array_equal(c.codes(w)[b, :, rows].cpu().numpy(),
                                              e[w + "_codes"][:, t0:t1]), (step, r, b, fid, w)
                        assert np.array_equal(c.scales(w)[b, :, rows].cpu().numpy(),
                                              e[w + "_scales"][:, t0:t1]), (step, r, b, fid, w)
