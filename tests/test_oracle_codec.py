"""Pins for the oracle's NVFP4 codec (CPU only).

The oracle's encoders are brute-force nearest searches; here they are checked
against things other than themselves:
  * library conversions: ml_dtypes float4_e2m1fn / float8_e4m3fn and
    torch.float8_e4m3fn (round-to-nearest-even casts);
  * closed forms: rounding to a 1- or 3-bit mantissa with numpy's
    half-to-even ``np.round``;
  * hand-derived blocks under tests/golden/;
  * exact round trips of every (code, scale) pair and format invariants.
"""
import json
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _floats_in_binades(lo_exp, hi_exp, stride=1):
    """All positive float32 values in [2^lo_exp, 2^hi_exp) (every stride-th)."""
    lo = np.float32(2.0 ** lo_exp).view(np.uint32)
    hi = np.float32(2.0 ** hi_exp).view(np.uint32)
    return np.arange(lo, hi, stride, dtype=np.uint32).view(np.float32)


# ------------------------------------------------------------------ decode

def test_e2m1_decode_matches_ml_dtypes():
    lib_vals = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    ours = np.array([oracle.e2m1_decode(c) for c in range(16)])
    assert np.array_equal(ours, lib_vals)


def test_e4m3_decode_matches_torch():
    lib_vals = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    ours = np.array([oracle.e4m3_decode(c) for c in range(256)])
    nan = np.isnan(lib_vals)
    assert np.array_equal(nan, np.isnan(ours)) and nan.sum() == 2
    assert np.array_equal(ours[~nan], lib_vals[~nan])


# ------------------------------------------------------------------ encode

def _ml_e2m1(y):
    c = np.asarray(y, np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    c[c == 8] = 0          # the cache stores no negative zero
    return c


@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_e2m1_encode_exhaustive_decision_range(sign):
    # every float in [2^-3, 2^4): all rounding decisions of E2M1 live here
    y = _floats_in_binades(-3, 4) * np.float32(sign)
    assert np.array_equal(oracle.e2m1_encode_array(y), _ml_e2m1(y))


def test_e2m1_encode_outside_decision_range():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 0x7F800000, size=2_000_000, dtype=np.uint32)
    y = bits.view(np.float32)
    y = np.concatenate([y, -y, np.float32([0.0, -0.0, 6.0, -6.0, 3.4e38, -3.4e38, 1e-45])])
    assert np.array_equal(oracle.e2m1_encode_array(y), _ml_e2m1(y))


def _closed_form_e2m1(y):
    """Round |y| to the E2M1 grid with numpy's half-to-even rounding."""
    a = np.abs(y.astype(np.float64))
    out = np.empty_like(a)
    sub = a < 1.0
    out[sub] = np.round(a[sub] * 2.0) / 2.0                     # spacing 0.5 below 1
    e = np.floor(np.log2(np.where(sub, 1.0, a)))
    e = np.minimum(e, 2.0)
    out[~sub] = np.round(a[~sub] / 2.0 ** e[~sub] * 2.0) / 2.0 * 2.0 ** e[~sub]
    return np.minimum(out, 6.0)


def test_e2m1_encode_matches_closed_form():
    y = _floats_in_binades(-4, 4, stride=97)
    codes = oracle.e2m1_encode_array(y)
    got = np.array([oracle.e2m1_decode(c) for c in range(16)])[codes]
    assert np.array_equal(got, _closed_form_e2m1(y))


def _torch_e4m3(t):
    return torch.from_numpy(np.ascontiguousarray(t, np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


def test_block_scale_code_vs_torch_near_every_grid_point():
    # every E4M3 value and midpoint, +-256 float ulps around each
    vals = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    mids = (vals[1:] + vals[:-1]) / 2
    pts = np.concatenate([vals, mids]).astype(np.float32)
    bits = pts.view(np.uint32).astype(np.int64)
    off = np.arange(-256, 257, dtype=np.int64)
    t = (bits[:, None] + off[None, :]).reshape(-1)
    t = t[(t >= 0) & (t < 0x7F800000)].astype(np.uint32).view(np.float32)
    t = t[t <= 448.0]
    assert np.array_equal(oracle.block_scale_code_array(t), _torch_e4m3(t))


def test_block_scale_code_vs_ml_dtypes_strided():
    t = _floats_in_binades(-12, 9, stride=101)
    t = t[t <= 448.0]
    lib_codes = t.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(oracle.block_scale_code_array(t), lib_codes)


def test_block_scale_clamps_at_448():
    t = np.float32([448.0, 448.00003, 464.0, 500.0, 1e6, 3.4e38])
    assert (oracle.block_scale_code_array(t) == 0x7E).all()


def _closed_form_e4m3(t):
    a = t.astype(np.float64)
    out = np.empty_like(a)
    sub = a < 2.0 ** -6
    out[sub] = np.round(a[sub] * 2.0 ** 9) / 2.0 ** 9
    e = np.floor(np.log2(np.where(sub, 1.0, a)))
    out[~sub] = np.round(a[~sub] / 2.0 ** e[~sub] * 8.0) / 8.0 * 2.0 ** e[~sub]
    return np.minimum(out, 448.0)


def test_block_scale_code_matches_closed_form():
    t = _floats_in_binades(-12, 9, stride=1009)
    t = t[t < 448.0]
    codes = oracle.block_scale_code_array(t)
    got = np.array([oracle.e4m3_decode(c) for c in range(127)])[codes]
    assert np.array_equal(got, _closed_form_e4m3(t))


# ------------------------------------------------------------------ blocks

def test_golden_blocks():
    with open(os.path.join(GOLDEN, "nvfp4_blocks.json")) as f:
        data = json.load(f)
    for blk in data["blocks"]:
        codes, scale = oracle.quantize_block16(np.float32(blk["x"]), blk["s_g"])
        assert scale == blk["scale"], blk["name"]
        assert codes.tolist() == blk["codes"], blk["name"]


def test_roundtrip_every_code_and_scale():
    # s_g = 2^-10 (a first-chunk amax of 2.625); a block holding all 16 codes at
    # scale s_b reproduces s_b and the codes (negative zero comes back as 0x0)
    s_g = oracle.global_scale(2.625)
    assert s_g == 2.0 ** -10
    e2m1 = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    e4m3 = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    want = np.arange(16, dtype=np.uint8)
    want[8] = 0
    for sb_code in range(1, 127):
        x = (e2m1 * e4m3[sb_code] * s_g).astype(np.float32)
        assert np.array_equal(x.astype(np.float64), e2m1 * e4m3[sb_code] * s_g)   # exact
        codes, scale = oracle.quantize_block16(x, s_g)
        assert scale == sb_code
        got = np.empty(16, np.uint8)
        got[0::2] = codes & 0xF
        got[1::2] = codes >> 4
        assert np.array_equal(got, want), sb_code


def test_amax_element_takes_code_six():
    # with a normal-range block scale the amax element always lands on +-6
    rng = np.random.default_rng(7)
    for _ in range(2000):
        x = (rng.standard_normal(16) * 10.0 ** rng.uniform(-2, 2)).astype(np.float32)
        s_g = np.float32(10.0 ** rng.uniform(-4, -1))
        codes, scale = oracle.quantize_block16(x, s_g)
        if scale < 0x08 or scale == 0x7E:       # subnormal or clamped scale
            continue
        q = np.empty(16, np.uint8)
        q[0::2] = codes & 0xF
        q[1::2] = codes >> 4
        i = int(np.argmax(np.abs(x)))
        assert q[i] & 7 == 7


def test_power_of_two_scale_invariance():
    rng = np.random.default_rng(3)
    for _ in range(500):
        x = rng.standard_normal(16).astype(np.float32)
        s_g = np.float32(rng.uniform(1e-3, 1e-2))
        base = oracle.quantize_block16(x, s_g)
        for k in (-3, -1, 2, 5):
            f = np.float32(2.0 ** k)
            other = oracle.quantize_block16(x * f, s_g * f)
            assert other[1] == base[1] and np.array_equal(other[0], base[0])


def test_dequant_error_bound():
    # |x - deq(x)| <= half the E2M1 grid spacing at |y|, times s_b*s_g, unless
    # the element saturated
    rng = np.random.default_rng(11)
    x = rng.standard_normal((256, 128)).astype(np.float32)
    s_g = oracle.global_scale(oracle.amax(x))
    codes, scales = oracle.quantize_rows(x, s_g)
    deq = oracle.dequant_rows(codes, scales, s_g)
    sb = np.array([oracle.e4m3_decode(c) for c in range(256)])[scales]
    d = np.repeat(sb, 16, axis=1) * np.float64(s_g)
    y = np.abs(x / d)
    half = np.where(y < 2, 0.25, np.where(y < 4, 0.5, 1.0))
    ok = (np.abs(deq - x) <= half * d * (1 + 1e-6)) | (y > 6)
    assert ok.all()


def test_global_scale_cases():
    assert oracle.global_scale(0.0) == 1.0
    assert oracle.global_scale(2688.0) == 1.0
    assert oracle.global_scale(2.625) == 2.0 ** -10
    assert oracle.global_scale(5376.0) == 2.0
    assert oracle.global_scale(1e-40) == 1.0          # would be subnormal
