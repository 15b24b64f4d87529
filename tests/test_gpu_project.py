"""K/V projection on the tensor cores and its fused quantize-append.

With small-integer inputs every partial sum is an fp32 value, so the GPU's
products are exact whatever its summation order: the bf16 K/V of
nvkv_kv_project must equal the oracle's bit for bit, and the fused
nvfp4_kv_project_append must leave the cache exactly as the oracle's
quantize-append of those K/V (and as project + append on the GPU), on the
first chunk (two-launch path) and later ones (fused epilogue).  With
Gaussian inputs the GPU's fp32 summation order may move a value across a
bf16 rounding boundary: at most 1 ulp, on a small fraction of values; the
fused and two-launch GPU paths still agree byte for byte."""
import numpy as np
import pytest
import torch

import kvsynth
from oracle.project import kv_project
from oracle.stream import OracleStream
from tests._harness import LibStream, assert_parity, sample_rows

pytestmark = pytest.mark.gpu


def _exact_inputs(wl, hidden, step):
    # x = i/4, w = j/2^s with |i|, |j| <= 8: every partial sum is a multiple
    # of 2^-(s+2) below 2^17 of them, an fp32 value; 2^s ~ 8 sqrt(hidden)
    # keeps K and V near unit scale
    s = 3 + int(np.ceil(np.log2(np.sqrt(hidden))))
    g = torch.Generator().manual_seed(1000 + step)
    x = (torch.randint(-8, 9, (wl.B, wl.Lq, hidden), generator=g) / 4).to(torch.bfloat16)
    wk = (torch.randint(-8, 9, (wl.H * 128, hidden), generator=g) / 2 ** s).to(torch.bfloat16)
    wv = (torch.randint(-8, 9, (wl.H * 128, hidden), generator=g) / 2 ** s).to(torch.bfloat16)
    return x, wk, wv


def _oracle_kv(x, w, wl):
    y = kv_project(x.float().numpy().reshape(-1, x.shape[-1]), w.float().numpy())
    return torch.from_numpy(y).reshape(wl.B, wl.Lq, wl.H, 128).to(torch.bfloat16)


def _make_room(cache):
    need = cache.desc.C - min(cache.free_frames(b) for b in range(cache.desc.B))
    if need > 0:
        cache.evict(need)


@pytest.mark.parametrize("name,hidden", [("tiny", 128), ("stream5b", 512), ("stream1p3b", 1536)])
def test_fused_projection_append_bit_exact(name, hidden):
    import nvfp4_kv_cache_append_b200 as nv
    wl = kvsynth.WORKLOADS[name]
    fused = LibStream(wl, nv.NVKV_KV_NVFP4)
    two = nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, nv.NVKV_KV_NVFP4)
    ora = OracleStream(wl, seed=0, keep_inputs=False)
    for step in range(1, 4):
        x, wk, wv = _exact_inputs(wl, hidden, step)
        kref, vref = _oracle_kv(x, wk, wl), _oracle_kv(x, wv, wl)
        q = kvsynth.chunk_qkv(wl, step, 0, which="q")["q"]
        new = ora.step(k=kref, v=vref, q=q)
        gx, gk, gv, gq = x.cuda(), wk.cuda(), wv.cuda(), q.cuda()
        _make_room(fused.cache)
        fused.cache.project_append(gx, gk, gv)
        lse = torch.empty(wl.B, wl.H, wl.Lq, device="cuda")
        out = fused.cache.attention(gq, lse=lse)
        _make_room(two)
        k, v = two.project(gx, gk, gv)
        two.append(k, v)
        torch.cuda.synchronize()
        assert fused.cache.device_status() == 0 and two.device_status() == 0
        assert torch.equal(k.cpu(), kref) and torch.equal(v.cpu(), vref)
        assert np.array_equal(fused.cache.global_scales().cpu().numpy(), ora.s_g)
        for b in range(wl.B):
            for fid in new[b]:
                rows = fused.frame_rows(b, fid)
                e = ora.frame(b, fid)
                for w in ("k", "v"):
                    got_c = fused.cache.codes(w)[b, :, rows].cpu().numpy()
                    assert np.array_equal(got_c, e[w + "_codes"]), (step, b, fid, w)
                    assert np.array_equal(fused.cache.scales(w)[b, :, rows].cpu().numpy(),
                                          e[w + "_scales"]), (step, b, fid, w)
        for w in ("k", "v"):
            assert torch.equal(fused.cache.codes(w), two.codes(w))
            assert torch.equal(fused.cache.scales(w), two.scales(w))
        got = out.float().cpu().numpy()
        rows = sample_rows(wl.Lq, 12, step)
        for h in range(0, wl.H, max(1, wl.H // 3)):
            ref, ref_lse = ora.attention(0, h, rows)
            assert_parity(got[0, rows, h], ref, f"step {step} h {h}")


def test_projection_gaussian_inputs():
    import nvfp4_kv_cache_append_b200 as nv
    wl = kvsynth.WORKLOADS["stream5b"]
    hidden = 1024
    g = torch.Generator().manual_seed(7)
    fused = nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, nv.NVKV_KV_NVFP4)
    two = nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, nv.NVKV_KV_NVFP4)
    for step in range(1, 4):
        x = torch.randn(wl.B, wl.Lq, hidden, generator=g).to(torch.bfloat16)
        wk = (torch.randn(wl.H * 128, hidden, generator=g) / hidden ** 0.5).to(torch.bfloat16)
        wv = (torch.randn(wl.H * 128, hidden, generator=g) / hidden ** 0.5).to(torch.bfloat16)
        gx, gk, gv = x.cuda(), wk.cuda(), wv.cuda()
        for c in (fused, two):
            _make_room(c)
        fused.project_append(gx, gk, gv)
        k, v = two.project(gx, gk, gv)
        two.append(k, v)
        torch.cuda.synchronize()
        for got, w in ((k, wk), (v, wv)):
            ref = _oracle_kv(x, w, wl).float()
            d = (got.cpu().float() - ref).abs()
            ulp = torch.maximum(ref.abs(), torch.full_like(ref, 2.0 ** -126)).log2().floor()
            ulp = torch.exp2(ulp - 7)
            # one bf16 ulp, plus the fp32 summation error where the sum
            # nearly cancels (values are of unit scale)
            assert (d <= ulp + 2e-5).all(), d.max()
            assert (d > 0).float().mean().item() < 1e-3
        for w in ("k", "v"):
            assert torch.equal(fused.codes(w), two.codes(w))
            assert torch.equal(fused.scales(w), two.scales(w))
        assert torch.equal(fused.global_scales(), two.global_scales())


def test_projection_rejects_bad_arguments():
    import nvfp4_kv_cache_append_b200 as nv
    from nvfp4_kv_cache_append_b200 import _lib as L
    wl = kvsynth.WORKLOADS["tiny"]
    c = nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, nv.NVKV_KV_NVFP4)
    x = torch.zeros(wl.B, wl.Lq, 96, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(wl.H * 128, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.NvkvError):          # hidden not a multiple of 64
        c.project(x, w, w)
    x = torch.zeros(wl.B, wl.Lq, 128, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(wl.H * 128, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.NvkvError):          # the first append needs scratch
        L.nvfp4_kv_project_append(c.desc, c.cache, c.ring, x.data_ptr(), 128, w.data_ptr(),
                                  w.data_ptr(), None, 0, None)
    t = nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, nv.NVKV_KV_BF16)
    with pytest.raises(ValueError):
        t.project_append(x, w, w)
    s = nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, nv.NVKV_KV_NVFP4,
                   shard_rank=1, shard_count=2)
    with pytest.raises(L.NvkvError):          # shards: not supported
        s.project(x, w, w)
    assert c.ring.steps == 0


def test_projection_odd_heads_two_streams():
    # H = 3: a 256-channel tile holds K head 2 and V head 0; B = 2: one row
    # tile spans both streams; T = 20 tokens, hidden = 64 (one stage per tile)
    import nvfp4_kv_cache_append_b200 as nv
    wl = kvsynth.Workload("oddh", B=2, H=3, D=128, grid_h=4, grid_w=5, C=2, S=1, W=3, steps=4)
    fused = LibStream(wl, nv.NVKV_KV_NVFP4)
    ora = OracleStream(wl, seed=0, keep_inputs=False)
    for step in range(1, wl.steps + 1):
        x, wk, wv = _exact_inputs(wl, 64, step)
        kref, vref = _oracle_kv(x, wk, wl), _oracle_kv(x, wv, wl)
        q = kvsynth.chunk_qkv(wl, step, 0, which="q")["q"]
        new = ora.step(k=kref, v=vref, q=q)
        k, v = fused.cache.project(x.cuda(), wk.cuda(), wv.cuda())
        _make_room(fused.cache)
        fused.cache.project_append(x.cuda(), wk.cuda(), wv.cuda())
        torch.cuda.synchronize()
        assert fused.cache.device_status() == 0
        assert torch.equal(k.cpu(), kref) and torch.equal(v.cpu(), vref)
        for b in range(wl.B):
            for fid in new[b]:
                rows = fused.frame_rows(b, fid)
                e = ora.frame(b, fid)
                for w in ("k", "v"):
                    assert np.array_equal(fused.cache.codes(w)[b, :, rows].cpu().numpy(),
                                          e[w + "_codes"]), (step, b, fid, w)
                    assert np.array_equal(fused.cache.scales(w)[b, :, rows].cpu().numpy(),
                                          e[w + "_scales"]), (step, b, fid, w)
