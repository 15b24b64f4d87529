"""Chunk attention parity against the fp64 oracle (run on the same dequantized
K/V and bf16 Q): max-abs <= 3e-2 and relative L2 <= 1e-2, for the NVFP4 cache
and the bf16-KV twin, on the tiny workload (every row), the streaming
workloads at full size after the ring wrapped (sampled rows spanning Q tiles
and the ragged tail) and the multi-shot batch."""
import numpy as np
import pytest
import torch

import kvsynth
from oracle.stream import OracleStream
from tests._harness import LibStream, assert_parity, sample_rows, to_gpu

pytestmark = pytest.mark.gpu


def _run(wl, kv_dtype, check_steps, rows_fn, heads_fn, sched=None):
    lib = LibStream(wl, kv_dtype, sched=sched)
    ora = OracleStream(wl, seed=0, shot_sched=sched if sched is not None else None,
                       keep_inputs=True)
    quantized = kv_dtype == 0
    worst = (0.0, 0.0)
    for step in range(1, max(check_steps) + 1):
        x = kvsynth.chunk_qkv(wl, step, 0)
        ora.step(k=x["k"], v=x["v"], q=x["q"])
        g = to_gpu(x)
        out, lse = lib.step(g["q"], g["k"], g["v"])
        torch.cuda.synchronize()
        assert lib.cache.device_status() == 0
        if step not in check_steps:
            continue
        got = out.float().cpu().numpy()
        glse = lse.cpu().numpy()
        for b in range(wl.B):
            for h in heads_fn(wl, step, b):
                rows = rows_fn(wl, step, b, h)
                ref, ref_lse = ora.attention(b, h, rows, quantized=quantized)
                ma, rl = assert_parity(got[b, rows, h, :], ref, f"step {step} b {b} h {h}")
                worst = (max(worst[0], ma), max(worst[1], rl))
                assert np.abs(glse[b, h, rows] - ref_lse).max() < 2e-2
    return worst


@pytest.mark.parametrize("kv_dtype", [0, 1], ids=["nvfp4", "bf16"])
def test_tiny_every_row(kv_dtype):
    wl = kvsynth.WORKLOADS["tiny"]
    _run(wl, kv_dtype, set(range(1, wl.steps + 1)),
         lambda wl, s, b, h: np.arange(wl.Lq), lambda wl, s, b: range(wl.H))


@pytest.mark.parametrize("kv_dtype", [0, 1], ids=["nvfp4", "bf16"])
def test_stream1p3b_full_size(kv_dtype):
    wl = kvsynth.WORKLOADS["stream1p3b"]
    _run(wl, kv_dtype, {1, wl.steps},
         lambda wl, s, b, h: sample_rows(wl.Lq, 12, 100 * s + h),
         lambda wl, s, b: range(wl.H))


@pytest.mark.parametrize("kv_dtype", [0, 1], ids=["nvfp4", "bf16"])
def test_stream5b_full_size(kv_dtype):
    wl = kvsynth.WORKLOADS["stream5b"]
    _run(wl, kv_dtype, {wl.steps},
         lambda wl, s, b, h: sample_rows(wl.Lq, 8, 100 * s + h),
         lambda wl, s, b: range(0, wl.H, 3))


def test_multishot_masks():
    wl = kvsynth.WORKLOADS["multishot"]
    sched = kvsynth.shot_schedule(wl, 0)
    # steps where shots have just changed for some batch element, and the end
    changes = sorted({i + 1 for s in sched for i in range(1, wl.steps) if s[i] != s[i - 1]})
    checks = set(changes[:3]) | {wl.steps}
    _run(wl, 0, checks, lambda wl, s, b, h: sample_rows(wl.Lq, 4, 7 * s + b + h),
         lambda wl, s, b: (b % wl.H, (b + 5) % wl.H), sched=sched)


def test_ragged_small_frames():
    # T = 20 tokens per frame (not a multiple of anything), C = 2: tiles mix
    # many frames and the last tile is ragged
    wl = kvsynth.Workload("odd", B=2, H=3, D=128, grid_h=4, grid_w=5, C=2, S=2, W=6, steps=6)
    _run(wl, 0, {1, 4, 6}, lambda wl, s, b, h: np.arange(wl.Lq), lambda wl, s, b: range(wl.H))


@pytest.mark.parametrize("kv_dtype", [0, 1], ids=["nvfp4", "bf16"])
def test_growing_logits_rescale(kv_dtype):
    """Keys of later frames grow step by step (x3 .. x6; the sink's chunk
    sets amax = 64 so that nothing saturates), so their logits sit more than
    2^8 above the sink's: the online softmax raises its running max between
    tiles and, with 192 tokens per frame, inside a tile that starts in the
    sink and ends in the window (P already written and O rescaled), and must
    still match the oracle on every row.  16 heads make 160 key tiles, so the
    persistent schedule gives each CTA pair segments of several tiles and the
    rescale of O between tiles runs too."""
    wl = kvsynth.Workload("grow", B=1, H=16, D=128, grid_h=16, grid_w=12, C=1, S=1, W=4, steps=5)
    lib = LibStream(wl, kv_dtype)
    ora = OracleStream(wl, seed=0, keep_inputs=True)
    quantized = kv_dtype == 0
    for step in range(1, wl.steps + 1):
        x = kvsynth.chunk_qkv(wl, step, 0)
        k = x["k"].float()
        if step == 1:
            k[0, 0, :, 0] = 64.0
        else:
            k = k * (1.0 + step)
        k = k.to(torch.bfloat16)
        ora.step(k=k, v=x["v"], q=x["q"])
        g = to_gpu({"q": x["q"], "k": k, "v": x["v"]})
        out, _ = lib.step(g["q"], g["k"], g["v"])
        torch.cuda.synchronize()
        assert lib.cache.device_status() == 0
        got = out.float().cpu().numpy()
        for h in range(wl.H):
            ref, _ = ora.attention(0, h, np.arange(wl.Lq), quantized=quantized)
            assert_parity(got[0, :, h], ref, f"step {step} h {h}")


def _scaled_run(wl, kv_dtype, qf, kf):
    """Outputs and LSE of every step of `wl` with Q times qf and K times kf,
    and the oracle's worst parity figures on every row."""
    lib = LibStream(wl, kv_dtype)
    ora = OracleStream(wl, seed=0, keep_inputs=True)
    outs = []
    for step in range(1, wl.steps + 1):
        x = kvsynth.chunk_qkv(wl, step, 0)
        q = (x["q"].float() * qf).to(torch.bfloat16)
        k = (x["k"].float() * kf).to(torch.bfloat16)
        ora.step(k=k, v=x["v"], q=q)
        g = to_gpu({"q": q, "k": k, "v": x["v"]})
        out, lse = lib.step(g["q"], g["k"], g["v"])
        torch.cuda.synchronize()
        assert lib.cache.device_status() == 0
        got = out.float().cpu().numpy()
        glse = lse.cpu().numpy()
        for h in range(wl.H):
            ref, ref_lse = ora.attention(0, h, np.arange(wl.Lq), quantized=kv_dtype == 0)
            assert_parity(got[0, :, h], ref, f"q x {qf} k x {kf} step {step} h {h}")
            assert np.abs(glse[0, h] - ref_lse).max() < 2e-2
        outs.append((out.cpu(), lse.cpu()))
    return outs


# Q scaled by an exact power of two, K by its inverse: the logits are the same
# real numbers (the NVFP4 quantization of K scales exactly with a power of
# two: s_g moves, the codes and block scales do not), so the NVFP4 call must
# return bit for bit what it returns on the unscaled inputs, and match the
# oracle.  At 2^+-40 the rotated Q lies far outside f16 (overflow, or
# subnormal loss) unless each row is range-scaled before the f16 rounding.
@pytest.mark.parametrize("e", [12, -12, 40, -40])
def test_q_range_compensated(e):
    wl = kvsynth.WORKLOADS["tiny"]
    base = _scaled_run(wl, 0, 1.0, 1.0)
    got = _scaled_run(wl, 0, 2.0 ** e, 2.0 ** -e)
    for (o0, l0), (o1, l1) in zip(base, got):
        assert torch.equal(o0, o1)
        assert torch.equal(l0, l1)


# Q alone times 2^-12 (logits 4096 times smaller: near-uniform attention) on
# both calls.  Q alone times 2^12 makes the softmax an argmax whose near-ties
# are decided by the last bit of the rotated Q, so the compensated form above
# stands in for it.
@pytest.mark.parametrize("kv_dtype", [0, 1], ids=["nvfp4", "bf16"])
def test_q_small(kv_dtype):
    _scaled_run(kvsynth.WORKLOADS["tiny"], kv_dtype, 2.0 ** -12, 1.0)


def test_q_large_bf16kv():
    """The twin with Q times 2^12 and K times 2^-12 (K stays inside f16)."""
    _scaled_run(kvsynth.WORKLOADS["tiny"], 1, 2.0 ** 12, 2.0 ** -12)


@pytest.mark.parametrize("kv_dtype", [0, 1], ids=["nvfp4", "bf16"])
def test_round_robin_schedule_with_split_tail(kv_dtype):
    """192 work items (2 streams x 32 heads x 3 query-tile pairs) of 14 key
    tiles on 74 CTA pairs: one round of whole items round-robin, then the
    other 118 items' tiles cut end to end, so that most of them are split
    between two pairs and merged through partial records.  Every row of
    sampled heads against the oracle."""
    wl = kvsynth.Workload("rr", B=2, H=32, D=128, grid_h=16, grid_w=16, C=3, S=1, W=6, steps=3)
    _run(wl, kv_dtype, {1, wl.steps}, lambda wl, s, b, h: np.arange(wl.Lq),
         lambda wl, s, b: range(b, wl.H, 5))
