"""The GPU pieces of the block-scaled FP4 Q K^T reading against the oracle:
the query side (every row quantized to NVFP4 once per visible key frame,
nvkv_fp4qk_quantize_q) bit for bit, over the ring's growth, wrap and
multi-shot masking.  (The key side, nvfp4_kv_append_spatial_rope, is checked
in test_gpu_append.py.)"""
import numpy as np
import pytest
import torch

import kvsynth
import oracle
from oracle.stream import OracleStream
from tests._harness import sample_rows, to_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,n_rows,heads", [("tiny", None, None), ("multishot", 6, (0, 7)),
                                               ("stream1p3b", 24, (0, 5, 11))])
def test_q_frames_bit_exact(name, n_rows, heads):
    import nvfp4_kv_cache_append_b200 as nv
    from nvfp4_kv_cache_append_b200 import _lib as L
    wl = kvsynth.WORKLOADS[name]
    sched = kvsynth.shot_schedule(wl, 9)
    cache = nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, nv.NVKV_KV_NVFP4)
    ora = OracleStream(wl, seed=9, keep_inputs=False, fp4_qk=True, shot_sched=sched)
    nv_max = wl.S + wl.W
    codes = torch.zeros(wl.B, wl.H, wl.Lq, nv_max, 64, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(wl.B, wl.H, wl.Lq, nv_max, 8, dtype=torch.uint8, device="cuda")
    sgq = torch.zeros(wl.B, wl.H, wl.Lq, dtype=torch.float32, device="cuda")
    steps = wl.steps if name == "tiny" else min(wl.steps, (wl.S + wl.W) // wl.C + 2)
    checks = set(range(1, steps + 1)) if name == "tiny" else {1, steps}
    for step in range(1, steps + 1):
        x = kvsynth.chunk_qkv(wl, step, 9)
        ora.step(k=x["k"], v=x["v"], q=x["q"])
        for b in range(wl.B):
            cache.begin_shot(b, sched[b][step - 1])
        need = wl.C - min(cache.free_frames(b) for b in range(wl.B))
        if need > 0:
            cache.evict(need)
        g = to_gpu(x)
        cache.append_spatial_rope(g["k"], g["v"])
        L.nvkv_fp4qk_quantize_q(cache.desc, cache.ring, g["q"].data_ptr(), codes.data_ptr(),
                                scales.data_ptr(), sgq.data_ptr())
        if step not in checks:
            continue
        torch.cuda.synchronize()
        assert cache.device_status() == 0
        gc, gs, gg = codes.cpu().numpy(), scales.cpu().numpy(), sgq.cpu().numpy()
        qf = x["q"].float().numpy()
        for b in range(wl.B):
            vis = list(ora.rings[b].visible())
            assert len(vis) == len(cache.visible(b)[2])
            qpos, qtok = ora.query_positions(b)
            rows = np.arange(wl.Lq) if n_rows is None else sample_rows(wl.Lq, n_rows, step + b)
            for h in (range(wl.H) if heads is None else heads):
                for r in rows:
                    row = np.ascontiguousarray(qf[b, r, h])
                    s = oracle.q_row_global_scale(row)
                    assert gg[b, h, r] == np.float32(s), (step, b, h, r)
                    for j, (fid, rank) in enumerate(vis):
                        c, sc = oracle.q_for_frame(row, int(qpos[r]) - rank, int(qtok[r]),
                                                   wl.grid_w, s)
                        assert np.array_equal(gc[b, h, r, j], c), (step, b, h, r, j)
                        assert np.array_equal(gs[b, h, r, j], sc), (step, b, h, r, j)


@pytest.mark.parametrize("name", ["tiny", "odd25"])
def test_fp4_logits_against_dequantized_products(name):
    """The block-scaled tensor-core contraction (nvkv_fp4qk_scores): every
    logit of every row against every visible key equals the oracle's block
    form of the FP4 dot product (fp64) to f32 rounding, at every step of the
    stream (ring growth and wrap)."""
    import nvfp4_kv_cache_append_b200 as nv
    from nvfp4_kv_cache_append_b200 import _lib as L
    wl = (kvsynth.Workload("odd25", B=2, H=2, D=128, grid_h=5, grid_w=5, C=2, S=1, W=4, steps=5)
          if name == "odd25" else kvsynth.WORKLOADS[name])
    cache = nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, nv.NVKV_KV_NVFP4)
    ora = OracleStream(wl, seed=11, keep_inputs=False, fp4_qk=True)
    mv = wl.S + wl.W
    codes = torch.zeros(wl.B, wl.H, wl.Lq, mv, 64, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(wl.B, wl.H, wl.Lq, mv, 8, dtype=torch.uint8, device="cuda")
    sgq = torch.zeros(wl.B, wl.H, wl.Lq, dtype=torch.float32, device="cuda")
    out = torch.full((wl.B, wl.H, wl.Lq, mv, wl.T), float("nan"), device="cuda")
    for step in range(1, wl.steps + 1):
        x = kvsynth.chunk_qkv(wl, step, 11)
        ora.step(k=x["k"], v=x["v"], q=x["q"])
        need = wl.C - min(cache.free_frames(b) for b in range(wl.B))
        if need > 0:
            cache.evict(need)
        g = to_gpu(x)
        cache.append_spatial_rope(g["k"], g["v"])
        L.nvkv_fp4qk_quantize_q(cache.desc, cache.ring, g["q"].data_ptr(), codes.data_ptr(),
                                scales.data_ptr(), sgq.data_ptr())
        L.nvkv_fp4qk_scores(cache.desc, cache.cache, cache.ring, codes.data_ptr(),
                            scales.data_ptr(), sgq.data_ptr(), out.data_ptr())
        torch.cuda.synchronize()
        assert cache.device_status() == 0
        got = out.cpu().numpy()
        qf = x["q"].float().numpy()
        for b in range(wl.B):
            vis = list(ora.rings[b].visible())
            qpos, qtok = ora.query_positions(b)
            for h in range(wl.H):
                sgk = float(ora.s_g[0, b, h])
                for r in range(wl.Lq):
                    row = np.ascontiguousarray(qf[b, r, h])
                    s = oracle.q_row_global_scale(row)
                    for j, (fid, rank) in enumerate(vis):
                        c, sc = oracle.q_for_frame(row, int(qpos[r]) - rank, int(qtok[r]),
                                                   wl.grid_w, s)
                        e = ora.frame(b, fid)
                        ref = np.array([oracle.fp4_dot(c, sc, s, e["k_codes"][h][i],
                                                       e["k_scales"][h][i], sgk)
                                        for i in range(wl.T)])
                        mag = max(1e-30, float(np.abs(ref).max()))
                        err = float(np.abs(got[b, h, r, j] - ref).max())
                        assert err <= 1e-5 * mag, (step, b, h, r, j, err, mag)
