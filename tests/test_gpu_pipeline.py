"""HostPipeline: host-in, host-out AR steps on three overlapped streams give
the same bytes as the plain device path, through evictions and shot changes,
with one pipeline or several sharing their streams."""
import pytest
import torch

import kvsynth
from tests._harness import to_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,n_pipes", [("tiny", 1), ("multishot", 1), ("stream5b", 3)])
def test_pipeline_matches_device_path(name, n_pipes):
    import nvfp4_kv_cache_append_b200 as nv
    wl = kvsynth.WORKLOADS[name]
    steps = min(wl.steps, 7)
    sched = kvsynth.shot_schedule(wl, 0) if wl.shots > 1 else None
    mk = lambda: nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, nv.NVKV_KV_NVFP4)
    streams = tuple(torch.cuda.Stream() for _ in range(3)) if n_pipes > 1 else None
    pipes = [nv.HostPipeline(mk(), streams=streams) for _ in range(n_pipes)]
    refs = [mk() for _ in range(n_pipes)]
    hosts, outs, want = [], [], []
    for step in range(1, steps + 1):
        for p in range(n_pipes):
            x = kvsynth.chunk_qkv(wl, step, 10 * p)
            h = {k: v.pin_memory() for k, v in x.items()}
            o = torch.empty(h["q"].shape, dtype=torch.bfloat16).pin_memory()
            shot = [sched[b][step - 1] for b in range(wl.B)] if sched else None
            pipes[p].submit(h["q"], h["k"], h["v"], o, shot=shot)
            hosts.append(h)                      # keep the host buffers alive until the end
            outs.append(o)
            g = to_gpu(x)
            if shot:
                for b, sid in enumerate(shot):
                    refs[p].begin_shot(b, sid)
            want.append(refs[p].step(g["q"], g["k"], g["v"]).cpu())
    for p in pipes:
        p.synchronize()
    assert all(p.done(i) for p in pipes for i in range(steps))
    for i, (o, w) in enumerate(zip(outs, want)):
        assert torch.equal(o, w), i
    assert all(p.cache.device_status() == 0 for p in pipes)
