"""Denoising-step overwrite of the newest chunk (nvfp4_kv_overwrite /
bf16_kv_overwrite): codes and scales bit-exact with the oracle's in-place
overwrite on every resident frame, s_g fixed again while the first chunk is
the only chunk and kept afterwards, the ring untouched, and attention after
the overwrites within the tolerance of the other parity tests."""
import numpy as np
import pytest
import torch

import kvsynth
from oracle.stream import OracleStream
from tests._harness import LibStream, assert_parity, to_gpu

pytestmark = pytest.mark.gpu

DENOISE = 3          # overwrites per AR step after its append (a 4-step schedule)


def _resident_match(lib, ora, wl):
    for b in range(wl.B):
        for fid in ora.rings[b].resident():
            rows = lib.frame_rows(b, fid)
            e = ora.frame(b, fid)
            for w in ("k", "v"):
                assert np.array_equal(lib.cache.codes(w)[b, :, rows].cpu().numpy(),
                                      e[w + "_codes"]), (b, fid, w)
                assert np.array_equal(lib.cache.scales(w)[b, :, rows].cpu().numpy(),
                                      e[w + "_scales"]), (b, fid, w)


@pytest.mark.parametrize("name", ["tiny", "stream5b"])
def test_overwrite_bit_exact_and_attention(name):
    import nvfp4_kv_cache_append_b200 as nv
    wl = kvsynth.WORKLOADS[name]
    lib = LibStream(wl, nv.NVKV_KV_NVFP4)
    ora = OracleStream(wl, seed=0, keep_inputs=False)
    steps = min(wl.steps, 5)
    for step in range(1, steps + 1):
        x = kvsynth.chunk_qkv(wl, step, 0)
        ora.step(k=x["k"], v=x["v"], q=x["q"])
        g = to_gpu(x)
        lib.step(g["q"], g["k"], g["v"])
        ring_before = bytes(lib.cache.ring)
        for d in range(1, DENOISE + 1):
            y = kvsynth.chunk_qkv(wl, step + 1000 * d, 0)
            ora.overwrite(k=y["k"], v=y["v"], q=y["q"])
            gy = to_gpu(y)
            lib.cache.overwrite(gy["k"], gy["v"])
            out = lib.cache.attention(gy["q"])
        torch.cuda.synchronize()
        assert bytes(lib.cache.ring) == ring_before
        assert lib.cache.device_status() == 0
        assert np.array_equal(lib.cache.global_scales().cpu().numpy(), ora.s_g), step
        _resident_match(lib, ora, wl)
        got = out.float().cpu().numpy()
        rows = np.unique(np.r_[0, 1, wl.Lq // 2, wl.Lq - 1, np.arange(0, wl.Lq, max(1, wl.Lq // 16))])
        for h in range(0, wl.H, max(1, wl.H // 4)):
            ref, _ = ora.attention(0, h, rows)
            assert_parity(got[0, rows, h], ref, f"step {step} h {h}")


def test_overwrite_bf16_twin_copies_exactly():
    import nvfp4_kv_cache_append_b200 as nv
    wl = kvsynth.WORKLOADS["tiny"]
    lib = LibStream(wl, nv.NVKV_KV_BF16)
    for step in range(1, 4):
        g = to_gpu(kvsynth.chunk_qkv(wl, step, 0))
        lib.step(g["q"], g["k"], g["v"], with_lse=False)
        y = kvsynth.chunk_qkv(wl, step + 1000, 0)
        gy = to_gpu(y)
        lib.cache.overwrite(gy["k"], gy["v"])
        torch.cuda.synchronize()
        rows = lib.frame_rows(0, step - 1)
        for w in ("k", "v"):
            want = y[w][0].transpose(0, 1).contiguous()
            got = lib.cache.codes(w)[0, :, rows].cpu()
            assert torch.equal(got.view(torch.int16), want.view(torch.int16))


def test_overwrite_before_any_append_is_rejected():
    import nvfp4_kv_cache_append_b200 as nv
    wl = kvsynth.WORKLOADS["tiny"]
    cache = nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, nv.NVKV_KV_NVFP4)
    z = torch.zeros(wl.B, wl.Lq, wl.H, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nv.NvkvError):
        cache.overwrite(z, z)
