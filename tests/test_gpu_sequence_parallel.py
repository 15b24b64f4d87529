"""Sequence-parallel KV split on one GPU: the shards of one cache run side by
side as separate caches (what each GPU of a split holds), fed the same whole
chunks.  Checked against the oracle: every shard's codes and scales bit-exact
with the oracle's whole-frame codes for its tokens; every shard's partial
attention and lse against the oracle's attention over those tokens; the
nvkv_lse_merge of the shards against the oracle's whole-cache attention; and
the merge of a query sub-range equal to the same rows of the full merge."""
import numpy as np
import pytest
import torch

import kvsynth
from oracle.merge import lse_merge as oracle_lse_merge
from oracle.merge import shard_tokens
from oracle.stream import OracleStream
from tests._harness import assert_parity, sample_rows, to_gpu

pytestmark = pytest.mark.gpu


def _slot_of(cache, b, fid):
    st = cache.ring.s[b]
    for i in range(st.n_resident):
        if st.frame[i] == fid:
            return st.slot[i]
    raise KeyError(fid)


# 60 tokens per frame in 4 shards: 15 per shard, an odd count, so every slot
# carries a padding row; 25 tokens per frame: an odd whole cache
ODD60 = kvsynth.Workload("odd60", B=2, H=3, D=128, grid_h=6, grid_w=10, C=2, S=1, W=6, steps=6)
ODD25 = kvsynth.Workload("odd25", B=1, H=2, D=128, grid_h=5, grid_w=5, C=1, S=1, W=4, steps=7)


@pytest.mark.parametrize("name,count,kv,steps", [
    ("tiny", 2, "nvfp4", 6), ("tiny", 4, "nvfp4", 6), ("tiny", 8, "bf16", 6),
    ("stream5b", 2, "nvfp4", 4), ("stream5b", 4, "bf16", 3), ("stream1p3b", 4, "nvfp4", 3),
    # 8 shards of the 1.3B-like stream: 195 tokens per shard (odd)
    ("stream1p3b", 8, "nvfp4", 2),
    (ODD60, 4, "nvfp4", 6), (ODD60, 4, "bf16", 4), (ODD25, 1, "nvfp4", 7)],
    ids=lambda v: v.name if isinstance(v, kvsynth.Workload) else None)
def test_shards_bit_exact_and_merge_to_whole_attention(name, count, kv, steps):
    import nvfp4_kv_cache_append_b200 as nv
    wl = name if isinstance(name, kvsynth.Workload) else kvsynth.WORKLOADS[name]
    dtype = nv.NVKV_KV_NVFP4 if kv == "nvfp4" else nv.NVKV_KV_BF16
    shards = [nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, dtype,
                         shard_rank=r, shard_count=count) for r in range(count)]
    ts = wl.T // count
    tr = ts + (ts & 1)                    # rows per slot: one padding row if ts is odd
    assert all(c.rows == (wl.S + wl.W) * tr for c in shards)
    ora = OracleStream(wl, seed=2, keep_inputs=(kv == "bf16"))
    quantized = kv == "nvfp4"
    for step in range(1, steps + 1):
        x = kvsynth.chunk_qkv(wl, step, 2)
        new = ora.step(k=x["k"], v=x["v"], q=x["q"])
        g = to_gpu(x)
        outs, lses = [], []
        for c in shards:
            lse = torch.empty(wl.B, wl.H, wl.Lq, dtype=torch.float32, device="cuda")
            outs.append(c.step(g["q"], g["k"], g["v"], lse=lse))
            lses.append(lse)
        merged_lse = torch.empty(wl.B, wl.H, wl.Lq, dtype=torch.float32, device="cuda")
        merged = nv.lse_merge(outs, lses, lse_out=merged_lse)
        # rank 1's query slice alone (the last rows for one shard): the same
        # rows as the full merge, bit for bit
        q0, q1 = (wl.Lq // count, 2 * wl.Lq // count) if count > 1 else (wl.Lq // 2, wl.Lq)
        part = nv.lse_merge(outs, lses, q0, q1)
        torch.cuda.synchronize()
        assert all(c.device_status() == 0 for c in shards)
        assert torch.equal(part, merged[:, q0:q1])
        for r, c in enumerate(shards):
            t0, t1 = shard_tokens(wl.T, count, r)
            if quantized:
                assert np.array_equal(c.global_scales().cpu().numpy(), ora.s_g)
            for b in range(wl.B):
                for fid in new[b]:
                    p = _slot_of(c, b, fid)
                    e = ora.frame(b, fid)
                    rows = slice(p * tr, p * tr + ts)
                    if quantized:
                        for w in ("k", "v"):
                            assert np.array_equal(c.codes(w)[b, :, rows].cpu().numpy(),
                                                  e[w + "_codes"][:, t0:t1]), (r, fid, w)
                            assert np.array_equal(c.scales(w)[b, :, rows].cpu().numpy(),
                                                  e[w + "_scales"][:, t0:t1]), (r, fid, w)
                    else:
                        for w in ("k", "v"):
                            assert np.array_equal(c.codes(w)[b, :, rows].float().cpu().numpy(),
                                                  e[w + "_bf16"][:, t0:t1]), (r, fid, w)
        rows = sample_rows(wl.Lq, 24, step)
        got = merged.float().cpu().numpy()
        glse = merged_lse.cpu().numpy()
        parts = [(o.float().cpu().numpy(), l.cpu().numpy()) for o, l in zip(outs, lses)]
        for b in range(wl.B):
            for h in range(0, wl.H, max(1, wl.H // 3)):
                ref, ref_lse = ora.attention(b, h, rows, quantized=quantized)
                assert_parity(got[b, rows, h], ref, f"merged step {step} b {b} h {h}")
                assert np.abs(glse[b, h, rows] - ref_lse).max() < 2e-2
                ro, rl = [], []
                for r, (po, pl) in enumerate(parts):
                    sref, sref_lse = ora.attention(b, h, rows, quantized=quantized,
                                                   tokens=shard_tokens(wl.T, count, r))
                    assert_parity(po[b, rows, h], sref, f"shard {r} step {step} b {b} h {h}")
                    assert np.abs(pl[b, h, rows] - sref_lse).max() < 2e-2
                    ro.append(sref)
                    rl.append(sref_lse)
                # the oracle's merge of its own shards agrees with its whole attention
                mo, _ = oracle_lse_merge(ro, rl)
                np.testing.assert_allclose(mo, ref, rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("n", [1, 3, 16])
def test_merge_kernel_against_oracle(n):
    import nvfp4_kv_cache_append_b200 as nv
    B, Lq, H = 2, 301, 5
    gen = torch.Generator().manual_seed(n)
    o = [torch.randn(B, Lq, H, 128, generator=gen).to(torch.bfloat16) for _ in range(n)]
    lse = [torch.randn(B, H, Lq, generator=gen) * 4 for _ in range(n)]
    if n > 1:
        lse[1][0, :, ::3] = -float("inf")            # parts without keys on some rows
        o[1][0, ::3] = float("nan")                  # whose outputs must carry no weight
    lse[0][1, 2, 7] = -float("inf")
    if n == 1:
        o[0][1, 7, 2] = 0.0                          # a row with no keys at all: zeros
    out = nv.lse_merge([t.cuda() for t in o], [t.cuda() for t in lse],
                       lse_out=(lo := torch.empty(B, H, Lq, device="cuda")))
    torch.cuda.synchronize()
    ref_o, ref_l = oracle_lse_merge([t.float().numpy() for t in o],
                                    [t.permute(0, 2, 1).double().numpy() for t in lse])
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    # bf16 output rounding on top of f32 accumulation
    np.testing.assert_allclose(got, ref_o, rtol=1e-2, atol=1e-2)
    gl = lo.cpu().permute(0, 2, 1).numpy()
    fin = np.isfinite(ref_l)
    np.testing.assert_allclose(gl[fin], ref_l[fin], rtol=1e-5, atol=1e-5)
    assert np.all(np.isneginf(gl[~fin]))


def test_merge_rejects_bad_arguments():
    import nvfp4_kv_cache_append_b200 as nv
    from nvfp4_kv_cache_append_b200 import _lib as L
    o = torch.zeros(1, 8, 2, 128, dtype=torch.bfloat16, device="cuda")
    l = torch.zeros(1, 2, 8, device="cuda")
    out = torch.empty(1, 8, 2, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.NvkvError):
        L.nvkv_lse_merge([], [], 1, 2, 8, 0, 8, out.data_ptr())
    with pytest.raises(L.NvkvError):
        L.nvkv_lse_merge([o.data_ptr()] * 17, [l.data_ptr()] * 17, 1, 2, 8, 0, 8, out.data_ptr())
    with pytest.raises(L.NvkvError):
        L.nvkv_lse_merge([o.data_ptr()], [l.data_ptr()], 1, 2, 8, 5, 5, out.data_ptr())
    with pytest.raises(L.NvkvError):
        L.nvkv_lse_merge([o.data_ptr() + 2], [l.data_ptr()], 1, 2, 8, 0, 8, out.data_ptr())
    with pytest.raises(ValueError):
        nv.lse_merge([o], [l], 0, 8, out=torch.empty(1, 4, 2, 128, dtype=torch.bfloat16, device="cuda"))


def test_sequence_parallel_class_on_one_rank():
    """SequenceParallelKV through a one-rank NCCL group: symmetric buffer,
    barrier and the merge over the peer-pointer list; with one shard the
    merge returns the attention output unchanged."""
    import os
    import socket

    import torch.distributed as dist

    import nvfp4_kv_cache_append_b200 as nv
    from nvfp4_kv_cache_append_b200.sp import SequenceParallelKV
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        wl = kvsynth.WORKLOADS["tiny"]
        sp = SequenceParallelKV(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, nv.NVKV_KV_NVFP4)
        ref = nv.KVCache(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.C, wl.S, wl.W, nv.NVKV_KV_NVFP4)
        assert sp.plan.queries == (0, wl.Lq) and len(sp.ptrs) == 1
        for step in range(1, wl.steps + 1):
            g = to_gpu(kvsynth.chunk_qkv(wl, step, 5))
            got = sp.step(g["q"], g["k"], g["v"])
            want = ref.step(g["q"], g["k"], g["v"])
            torch.cuda.synchronize()
            assert torch.equal(got, want), step
        assert sp.cache.device_status() == 0
        del sp
    finally:
        dist.destroy_process_group()


def _merge_inputs(n, B=1, Lq=200, H=3, seed=0):
    gen = torch.Generator().manual_seed(seed)
    o = [torch.randn(B, Lq, H, 128, generator=gen).to(torch.bfloat16).cuda() for _ in range(n)]
    lse = [(torch.randn(B, H, Lq, generator=gen) * 3).cuda() for _ in range(n)]
    return o, lse


def test_synced_merge_after_peer_signal():
    """Rank 0 of 2, with rank 1's signal for epoch 1 already in rank 0's flag
    array (stored by the host, standing in for rank 1's kernel): the synced
    merge signals rank 1, passes the barrier and returns what the plain merge
    returns, bit for bit; the status stays 0."""
    import nvfp4_kv_cache_append_b200 as nv
    from nvfp4_kv_cache_append_b200 import _lib as L
    o, lse = _merge_inputs(2)
    B, Lq, H = 1, 200, 3
    flags = [torch.zeros(16, dtype=torch.int32, device="cuda") for _ in range(2)]
    flags[0][1] = 1
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty(B, 100, H, 128, dtype=torch.bfloat16, device="cuda")
    L.nvkv_lse_merge_synced([t.data_ptr() for t in o], [t.data_ptr() for t in lse],
                            [f.data_ptr() for f in flags], 0, 1, 2_000_000, status.data_ptr(),
                            B, H, Lq, 0, 100, out.data_ptr())
    want = nv.lse_merge(o, lse, 0, 100)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(out, want)
    assert flags[1][0].item() == 1 and flags[0][0].item() == 1     # rank 0 signalled both


def test_synced_merge_times_out_without_signal():
    """No rank 1 signal ever arrives: the wait runs out after 0.3 s, the kernel
    writes NVKV_ERR_TIMEOUT to the status word and returns; the context stays
    usable (a plain merge afterwards gives the right answer)."""
    import nvfp4_kv_cache_append_b200 as nv
    from nvfp4_kv_cache_append_b200 import _lib as L
    o, lse = _merge_inputs(2, seed=1)
    B, Lq, H = 1, 200, 3
    flags = [torch.zeros(16, dtype=torch.int32, device="cuda") for _ in range(2)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty(B, Lq, H, 128, dtype=torch.bfloat16, device="cuda")
    L.nvkv_lse_merge_synced([t.data_ptr() for t in o], [t.data_ptr() for t in lse],
                            [f.data_ptr() for f in flags], 0, 1, 300_000, status.data_ptr(),
                            B, H, Lq, 0, Lq, out.data_ptr())
    torch.cuda.synchronize()
    assert int(status.item()) == L.STATUS_CODE["NVKV_ERR_TIMEOUT"]
    assert flags[1][0].item() == 1                                 # the signal went out first
    again = nv.lse_merge(o, lse)
    ref_o, _ = oracle_lse_merge([t.float().cpu().numpy() for t in o],
                                [t.cpu().permute(0, 2, 1).double().numpy() for t in lse])
    torch.cuda.synchronize()
    np.testing.assert_allclose(again.float().cpu().numpy(), ref_o, rtol=1e-2, atol=1e-2)


def test_synced_merge_rejects_bad_arguments():
    from nvfp4_kv_cache_append_b200 import _lib as L
    o, lse = _merge_inputs(2)
    flags = [torch.zeros(16, dtype=torch.int32, device="cuda") for _ in range(2)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty(1, 200, 3, 128, dtype=torch.bfloat16, device="cuda")
    op, lp, fp = [t.data_ptr() for t in o], [t.data_ptr() for t in lse], [f.data_ptr() for f in flags]
    for rank, epoch, timeout, fl, st in [(2, 1, 1000, fp, status.data_ptr()),
                                         (0, 0, 1000, fp, status.data_ptr()),
                                         (0, 1, 0, fp, status.data_ptr()),
                                         (0, 1, 1000, [fp[0], 0], status.data_ptr()),
                                         (0, 1, 1000, fp, 0)]:
        with pytest.raises(L.NvkvError):
            L.nvkv_lse_merge_synced(op, lp, fl, rank, epoch, timeout, st, 1, 3, 200, 0, 200,
                                    out.data_ptr())
    with pytest.raises(L.NvkvError):
        L.nvkv_lse_merge_synced(op, lp, [fp[0] + 2, fp[1]], 0, 1, 1000, status.data_ptr(), 1, 3,
                                200, 0, 200, out.data_ptr())
    assert int(status.item()) == 0
