"""Long streaming run (1.3B-like shapes, 600 AR steps with ring eviction):
codes and scales match the oracle at steps 1, 10, 100 and 600, attention at
steps 100 and 600 matches on sampled rows of every head, the cache
footprint is constant and no device memory is allocated per step."""
import numpy as np
import pytest
import torch

import kvsynth
import oracle
from oracle.ring import OracleRing
from tests._harness import LibStream, assert_parity, sample_rows, to_gpu

pytestmark = pytest.mark.gpu

CHECK = (1, 10, 100, 600)


def test_long_run_600_steps():
    import nvfp4_kv_cache_append_b200 as nv
    wl = kvsynth.WORKLOADS["long600"]
    C, T = wl.C, wl.T
    MID = 100
    window = lambda s: set(range(s - wl.W // C + 1, s + 1))      # steps resident at step s
    oracle_steps = set(CHECK) | window(wl.steps) | window(MID)
    lib = LibStream(wl, nv.NVKV_KV_NVFP4)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(12345)
    ring = OracleRing(wl.S, wl.W, wl.C)
    kept = {}
    s_g = None
    mem0 = None
    free0 = None
    for step in range(1, wl.steps + 1):
        if step in oracle_steps:
            x = kvsynth.chunk_qkv(wl, step, 0)
            g = to_gpu(x)
        else:
            shape = (wl.B, wl.Lq, wl.H, 128)
            g = {n: torch.randn(shape, generator=gen, device="cuda").to(torch.bfloat16)
                 for n in "qkv"}
        out, _ = lib.step(g["q"], g["k"], g["v"], with_lse=False)
        new = ring.step()
        if step == MID:
            mid = (out.cpu(), ring.visible(), ring.query_pos0())      # host copy: no device memory
        if step == 1:
            xf = {n: x[n].float().numpy() for n in "kv"}
            s_g = np.array([[oracle.global_scale(oracle.amax(np.ascontiguousarray(xf[n][0, :, h])))
                             for h in range(wl.H)] for n in "kv"], np.float32)
        if step in oracle_steps:
            kept[step] = x
        if step in CHECK:
            torch.cuda.synchronize()
            for c, fid in enumerate(new):
                rows = lib.frame_rows(0, fid)
                for t, n in enumerate("kv"):
                    src = x[n][0, c * T:(c + 1) * T].float().numpy().transpose(1, 0, 2)
                    got_c = lib.cache.codes(n)[0, :, rows].cpu().numpy()
                    got_s = lib.cache.scales(n)[0, :, rows].cpu().numpy()
                    for h in range(wl.H):
                        codes, scales = oracle.quantize_rows(src[h], s_g[t, h])
                        assert np.array_equal(got_c[h], codes), (step, fid, n, h)
                        assert np.array_equal(got_s[h], scales), (step, fid, n, h)
        if step == 8:
            torch.cuda.synchronize()
            mem0 = torch.cuda.memory_allocated()
            free0 = torch.cuda.mem_get_info()[0]
            foot0 = lib.cache.footprint_bytes()
        if step > 8 and step % 97 == 0:
            torch.cuda.synchronize()
            del out
            assert torch.cuda.memory_allocated() <= mem0
            assert lib.cache.footprint_bytes() == foot0
    torch.cuda.synchronize()
    assert lib.cache.device_status() == 0
    assert torch.cuda.mem_get_info()[0] >= free0 - (64 << 20)
    assert ring.resident() == lib.cache.visible(0)[2]

    # attention at steps 100 and 600 on sampled rows of every head, from
    # regenerated inputs only
    fid_step = lambda fid: (fid // C + 1, fid % C)
    for at_step, got_out, visible, qpos0 in ((MID,) + mid, (wl.steps, out, ring.visible(),
                                                              ring.query_pos0())):
        q = kept[at_step]["q"][0]
        for h in range(wl.H):
            ks, vs, fpos, tok = [], [], [], []
            for fid, rank in visible:
                st, c = fid_step(fid)
                src = kept[st]
                for t, (n, lst) in enumerate((("k", ks), ("v", vs))):
                    rows_in = src[n][0, c * T:(c + 1) * T, h].float().numpy()
                    codes, scales = oracle.quantize_rows(rows_in, s_g[t, h])
                    lst.append(oracle.dequant_rows(codes, scales, s_g[t, h]))
                fpos.append(np.full(T, rank, np.int32))
                tok.append(np.arange(T, dtype=np.int32))
            l = np.arange(wl.Lq)
            qpos = (qpos0 + l // T).astype(np.int32)
            rows = sample_rows(wl.Lq, 12, 31 * at_step + h)
            ref, _ = oracle.attention_rows(q[:, h], np.concatenate(ks), np.concatenate(vs),
                                           np.concatenate(fpos), np.concatenate(tok), qpos,
                                           (l % T).astype(np.int32), rows, wl.grid_w)
            got = got_out[0, rows, h].float().cpu().numpy()
            assert_parity(got, ref, f"step {at_step} head {h}")
