"""The path at the limits of the C ABI: 16 streams, 64 heads, 64 resident
frames (the ring's maximum) with 16-frame chunks, through several evictions;
and the widest and tallest latent grids (256 columns, 256 rows), which size
the RoPE tables.  Codes and scales bit-exact, attention within the parity
bar on sampled streams, heads and rows."""
import numpy as np
import pytest
import torch

import kvsynth
from oracle.stream import OracleStream
from tests._harness import LibStream, assert_parity, to_gpu
from tests.test_gpu_attention import _run

pytestmark = pytest.mark.gpu


def test_maximum_streams_heads_frames_chunk():
    import nvfp4_kv_cache_append_b200 as nv
    wl = kvsynth.Workload("limits", B=16, H=64, D=128, grid_h=4, grid_w=4, C=16, S=4, W=60,
                          steps=6)
    lib = LibStream(wl, nv.NVKV_KV_NVFP4)
    ora = OracleStream(wl, seed=0, keep_inputs=False)
    for step in range(1, wl.steps + 1):
        x = kvsynth.chunk_qkv(wl, step, 0)
        new = ora.step(k=x["k"], v=x["v"], q=x["q"])
        g = to_gpu(x)
        out, lse = lib.step(g["q"], g["k"], g["v"])
        torch.cuda.synchronize()
        assert lib.cache.device_status() == 0
        if step == 1:
            assert np.array_equal(lib.cache.global_scales().cpu().numpy(), ora.s_g)
        codes = {w: lib.cache.codes(w).cpu().numpy() for w in ("k", "v")}
        scales = {w: lib.cache.scales(w).cpu().numpy() for w in ("k", "v")}
        for b in range(wl.B):
            assert lib.cache.ring.s[b].n_resident == len(ora.rings[b].resident())
            for fid in new[b]:
                rows = lib.frame_rows(b, fid)
                e = ora.frame(b, fid)
                for w in ("k", "v"):
                    assert np.array_equal(codes[w][b, :, rows], e[w + "_codes"]), (step, b, fid, w)
                    assert np.array_equal(scales[w][b, :, rows], e[w + "_scales"]), (step, b, fid, w)
        if step in (4, 6):                  # ring full (64 frames), then after evictions
            got = out.float().cpu().numpy()
            glse = lse.cpu().numpy()
            rows = np.arange(0, wl.Lq, 5)
            for b, h in [(0, 0), (7, 33), (15, 63)]:
                ref, ref_lse = ora.attention(b, h, rows)
                assert_parity(got[b, rows, h], ref, f"step {step} b {b} h {h}")
                assert np.abs(glse[b, h, rows] - ref_lse).max() < 2e-2


@pytest.mark.parametrize("grid", [(2, 256), (256, 2)], ids=["wide", "tall"])
@pytest.mark.parametrize("kv_dtype", [0, 1], ids=["nvfp4", "bf16"])
def test_largest_grids(grid, kv_dtype):
    wl = kvsynth.Workload("grid", B=1, H=2, D=128, grid_h=grid[0], grid_w=grid[1], C=1, S=1, W=3,
                          steps=5)
    _run(wl, kv_dtype, {2, 5}, lambda wl, s, b, h: np.arange(wl.Lq), lambda wl, s, b: range(wl.H))
