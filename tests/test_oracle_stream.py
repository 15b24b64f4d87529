"""Pins for the oracle's ring model and streaming pipeline (CPU only).

  * hand-traced ring sequences under tests/golden/ring_traces.json;
  * NVFP4-cache attention equals bf16-cache attention when every K/V value is
    exactly representable (quantization is then lossless);
  * poisoning frames that the mask hides leaves the output unchanged;
  * a multi-shot run whose batch has a single shot reduces to the plain
    streaming run.
"""
import json
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import kvsynth
import oracle
from oracle.ring import OracleRing
from oracle.stream import OracleStream

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _traces():
    with open(os.path.join(GOLDEN, "ring_traces.json")) as f:
        return json.load(f)["traces"]


@pytest.mark.parametrize("trace", _traces(), ids=lambda t: t["name"])
def test_ring_golden_trace(trace):
    ring = OracleRing(trace["S"], trace["W"], trace["C"])
    for i, shot in enumerate(trace["shots"]):
        ring.begin_shot(shot)
        ring.step()
        assert ring.resident() == trace["resident"][i], i
        assert [list(x) for x in ring.visible()] == trace["visible"][i], i
        assert ring.query_pos0() == trace["query_pos0"][i], i


def test_ring_errors():
    ring = OracleRing(1, 2, 1)
    ring.append(); ring.append(); ring.append()
    with pytest.raises(ValueError):
        ring.append()
    with pytest.raises(ValueError):
        ring.evict(3)
    assert ring.evict(2) == [1, 2]


def test_ring_footprint_constant_long_run():
    wl = kvsynth.WORKLOADS["long600"]
    ring = OracleRing(wl.S, wl.W, wl.C)
    for step in range(wl.steps):
        ring.step()
        if step >= 6:
            assert len(ring.resident()) == wl.S + wl.W
    assert ring.resident()[:3] == [0, 1, 2]
    assert ring.resident()[3:] == list(range(600 * 3 - 18, 600 * 3))


def _representable_chunk(wl, rng, first):
    """bf16 K/V whose every block is code * s_b * 2^-10 with a code of +-6 in it."""
    e2m1 = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    e4m3 = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    out = []
    for _ in range(2):
        n = wl.B * wl.Lq * wl.H * 8
        codes = rng.integers(0, 16, (n, 16))
        codes[:, 0] = rng.choice([7, 15], n)              # amax16 = 6 * s_b * s_g
        sb = e4m3[rng.integers(40, 127, n)]
        if first:
            sb[0] = 448.0                                  # first-chunk amax = 2.625
        x = e2m1[codes] * sb[:, None] * 2.0 ** -10
        out.append(torch.from_numpy(x.reshape(wl.B, wl.Lq, wl.H, 128)).to(torch.bfloat16))
    assert all(torch.equal(t.double(), torch.from_numpy(
        t.double().numpy())) for t in out)
    return out


def test_lossless_when_representable():
    wl = kvsynth.Workload("rep", B=1, H=2, D=128, grid_h=4, grid_w=4, C=1, S=1, W=2, steps=4)
    rng = np.random.default_rng(0)
    st = OracleStream(wl, seed=0)
    for step in range(4):
        k, v = _representable_chunk(wl, rng, first=(step == 0))
        q = kvsynth.chunk_qkv(wl, step + 1, 0)["q"]
        st.step(k=k, v=v, q=q)
        assert np.all(st.s_g == np.float32(2.0 ** -10))
        for h in range(wl.H):
            kq, vq, _, _ = st.visible_kv(0, h, quantized=True)
            kb, vb, _, _ = st.visible_kv(0, h, quantized=False)
            assert np.array_equal(kq, kb) and np.array_equal(vq, vb)
            rows = np.arange(wl.Lq)
            a, _ = st.attention(0, h, rows, quantized=True)
            b, _ = st.attention(0, h, rows, quantized=False)
            assert np.array_equal(a, b)


def test_masked_frames_do_not_leak():
    wl = kvsynth.Workload("ms", B=1, H=1, D=128, grid_h=2, grid_w=4, C=1, S=1, W=4, steps=9)
    sched = [[0, 0, 0, 1, 1, 1, 1, 2, 2]]
    st = OracleStream(wl, seed=5, shot_sched=sched)
    for _ in range(8):
        st.step()
    rows = np.arange(wl.Lq)
    ref, _ = st.attention(0, 0, rows)
    vis = {fid for fid, _ in st.rings[0].visible()}
    hidden = [fid for fid in st.rings[0].resident() if fid not in vis]
    assert hidden, "this schedule hides frames at step 8"
    for fid in hidden:
        e = st.store[(0, fid)]
        e["k_codes"][:] = 0x77
        e["v_codes"][:] = 0x77
        e["k_scales"][:] = 0x7E
        e["v_scales"][:] = 0x7E
    out, _ = st.attention(0, 0, rows)
    assert np.array_equal(out, ref)


def test_single_shot_multishot_reduces_to_stream():
    wl = kvsynth.Workload("s1", B=1, H=1, D=128, grid_h=2, grid_w=4, C=1, S=1, W=3, steps=6)
    a = OracleStream(wl, seed=2)
    b = OracleStream(wl, seed=2, shot_sched=[[0] * 6])
    rows = np.arange(wl.Lq)
    for _ in range(6):
        a.step(); b.step()
        assert np.array_equal(a.attention(0, 0, rows)[0], b.attention(0, 0, rows)[0])


def test_tiny_workload_stream_runs():
    wl = kvsynth.WORKLOADS["tiny"]
    st = OracleStream(wl, seed=0)
    for step in range(wl.steps):
        st.step()
        for h in range(wl.H):
            out, lse = st.attention(0, h, np.arange(wl.Lq))
            assert np.isfinite(out).all() and np.isfinite(lse).all()
    assert st.rings[0].resident() == [0, 3, 4, 5]


def test_shot_lengths_recipe():
    wl = kvsynth.WORKLOADS["multishot"]
    lens = kvsynth.shot_lengths(wl, 0)
    assert lens[0] == [8, 8, 8]
    for l in lens:
        assert sum(l) == 24 and len(l) == 3 and min(l) >= 2
    assert len({tuple(l) for l in lens}) > 1


@pytest.mark.parametrize("at_step", [1, 3, 6])
def test_overwrite_equals_append_of_the_new_values(at_step):
    """A denoising overwrite leaves the oracle stream exactly as if the chunk
    had been appended with the new values in the first place: same frames,
    same codes and scales, the same global scales (fixed again at step 1,
    kept afterwards) and the same attention."""
    wl = kvsynth.WORKLOADS["tiny"]
    a = OracleStream(wl, seed=0)
    b = OracleStream(wl, seed=0)
    for step in range(1, at_step + 1):
        x = kvsynth.chunk_qkv(wl, step, 0)
        if step < at_step:
            a.step(k=x["k"], v=x["v"], q=x["q"])
            b.step(k=x["k"], v=x["v"], q=x["q"])
            continue
        y = kvsynth.chunk_qkv(wl, step + 100, 0)       # the refined K/V of the same chunk
        a.step(k=x["k"], v=x["v"], q=x["q"])
        s_before = a.s_g.copy()
        new_a = a.overwrite(k=y["k"], v=y["v"], q=y["q"])
        new_b = b.step(k=y["k"], v=y["v"], q=y["q"])
        assert new_a == new_b
        if at_step > 1:
            assert np.array_equal(a.s_g, s_before)
    assert np.array_equal(a.s_g, b.s_g)
    assert a.rings[0].resident() == b.rings[0].resident()
    for fid in a.rings[0].resident():
        ea, eb = a.frame(0, fid), b.frame(0, fid)
        for key in ("k_codes", "k_scales", "v_codes", "v_scales"):
            assert np.array_equal(ea[key], eb[key]), (fid, key)
    for h in range(wl.H):
        oa, la = a.attention(0, h, np.arange(wl.Lq))
        ob, lb = b.attention(0, h, np.arange(wl.Lq))
        assert np.array_equal(oa, ob) and np.array_equal(la, lb)
