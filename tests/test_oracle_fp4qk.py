"""Pins of the oracle's block-scaled FP4 Q K^T reading (nvfp4_oracle.c, section
"block-scaled FP4 Q K^T (a reading)"), on the CPU.  What fixes each step:

- the split of the 3D RoPE between append (K's spatial pairs) and query (the
  frame pairs by the relative index): with Q kept in float and K' unquantized
  the FP4-path attention must equal the current path's fp64 attention to
  float rounding, on nontrivial positions (a wrong sign of the relative
  index, a swapped h/w or a dropped segment fails it by orders of magnitude);
- the float rotation: identity at position 0, norm kept and agreement with
  the fp64 rotation to a few float ulps, cos^2 + sin^2 = 1 to rounding;
- only relative frame indices enter: shifting every frame index by a
  constant leaves the FP4-path attention unchanged bit for bit;
- the per-row Q global scale: closed forms, and no Q_fk of any rotation
  saturates its block scales;
- the block form of the contraction equals the dot product of the
  dequantized rows (exact small-integer sums x scales);
- when every Q_fk is exactly representable (trivial rotations, values code x
  s_b x s_g), the FP4 path equals the current path."""
import numpy as np
import pytest

import kvsynth
import oracle
from oracle.stream import OracleStream


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16(x):
    import torch
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy()


# ------------------------------------------------------------ float rotation

def test_rope_f32_identity_at_zero_and_close_to_fp64():
    x = _bf16(_rng(1).standard_normal(128) * 3)
    assert np.array_equal(oracle.rope3d_f32(x, (0, 0, 0)), x)
    for pos in [(1, 0, 0), (0, 5, 0), (0, 0, 7), (17, 29, 51), (-3, 2, 1)]:
        got = oracle.rope3d_f32(x, pos).astype(np.float64)
        ref = oracle.rope3d(x.astype(np.float64), pos)
        pairs = np.hypot(x[0::2], x[1::2]).repeat(2)
        # two products and one sum in float, from float cos/sin: a few ulps
        assert np.all(np.abs(got - ref) <= 6 * 2.0 ** -24 * pairs + 1e-30), pos
        # the pair magnitudes are kept up to the same rounding
        np.testing.assert_allclose(np.hypot(got[0::2], got[1::2]), pairs[0::2], rtol=1e-6)


def test_rope_cs_f32_is_a_rounded_unit_vector():
    for d, n in [(44, 22), (42, 21)]:
        for i in range(n):
            for pos in [0, 1, 2, 7, 30, 255, -4]:
                c, s = oracle.rope_cs_f32(pos, i, d)
                assert abs(float(c) ** 2 + float(s) ** 2 - 1.0) < 4 * 2.0 ** -24
                if pos == 0:
                    assert (c, s) == (1.0, 0.0)
                c2, s2 = oracle.rope_cs_f32(-pos, i, d)
                assert c2 == c and s2 == -s                      # cos even, sin odd


def test_k_spatial_rope_leaves_the_frame_segment():
    k = _bf16(_rng(2).standard_normal((40, 128)))
    tok = np.arange(40, dtype=np.int32) * 3 + 1
    got = oracle.k_spatial_rope_f32(k, tok, grid_w=8)
    assert np.array_equal(got[:, :44], k[:, :44])
    for r in range(40):
        assert np.array_equal(got[r], oracle.rope3d_f32(k[r], (0, tok[r] // 8, tok[r] % 8)))
    assert not np.array_equal(got[:, 44:], k[:, 44:])


# ------------------------------------------------------------ the RoPE split

def _random_case(seed, Lk=96, Lq=12, grid_w=8, n_frames=6):
    g = _rng(seed)
    q = _bf16(g.standard_normal((Lq, 128)))
    k = _bf16(g.standard_normal((Lk, 128)))
    v = g.standard_normal((Lk, 128))
    kpos = g.integers(0, n_frames, Lk).astype(np.int32)
    ktok = g.integers(0, 64, Lk).astype(np.int32)
    qpos = g.integers(n_frames - 2, n_frames, Lq).astype(np.int32)
    qtok = g.integers(0, 64, Lq).astype(np.int32)
    return q, k, v, kpos, ktok, qpos, qtok, grid_w


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_rope_split_equals_full_rope_without_quantization(seed):
    q, k, v, kpos, ktok, qpos, qtok, gw = _random_case(seed)
    rows = np.arange(q.shape[0])
    ref, ref_lse = oracle.attention_rows(q, k.astype(np.float64), v, kpos, ktok, qpos, qtok, rows, gw)
    kp = oracle.k_spatial_rope_f32(k, ktok, gw).astype(np.float64)
    got, lse = oracle.attention_rows_fp4qk(q, kp, v, kpos, qpos, qtok, rows, gw, quantize_q=False)
    # float rotations only: logits agree to ~1e-6 relative
    np.testing.assert_allclose(got, ref, rtol=0, atol=2e-5)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=2e-5)
    # the same comparison with the frame index of the keys negated (a sign
    # error in the relative index) is far off: the check has teeth
    bad, _ = oracle.attention_rows_fp4qk(q, kp, v, -kpos + 2 * qpos.max(), qpos, qtok, rows, gw,
                                         quantize_q=False)
    assert np.abs(bad - ref).max() > 1e-2


def test_only_relative_frame_indices_enter():
    q, k, v, kpos, ktok, qpos, qtok, gw = _random_case(5)
    rows = np.arange(q.shape[0])
    kp = oracle.k_spatial_rope_f32(k, ktok, gw)
    s_g = oracle.global_scale(oracle.amax(kp))
    kc, ks = oracle.quantize_rows(kp, s_g)
    kd = oracle.dequant_rows(kc, ks, s_g)
    a, la = oracle.attention_rows_fp4qk(q, kd, v, kpos, qpos, qtok, rows, gw)
    b, lb = oracle.attention_rows_fp4qk(q, kd, v, kpos + 11, qpos + 11, qtok, rows, gw)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


# ------------------------------------------------------------ Q quantization

def test_q_row_global_scale_closed_forms():
    z = np.zeros(128, np.float32)
    assert oracle.q_row_global_scale(z) == 1.0
    x = z.copy()
    x[10], x[11] = 3.0, 4.0                          # one pair of magnitude 5
    assert oracle.q_row_global_scale(x) == float(np.float32(5.0 / 2688.0))
    x[100] = -12.0                                   # a larger pair (-12, 0)
    assert oracle.q_row_global_scale(x) == float(np.float32(12.0 / 2688.0))


@pytest.mark.parametrize("seed", [0, 3])
def test_no_rotation_saturates_the_q_block_scales(seed):
    g = _rng(seed)
    for _ in range(20):
        q = _bf16(g.standard_normal(128) * np.exp(g.uniform(-8, 8)))
        s = oracle.q_row_global_scale(q)
        for dpos in (-2, 0, 1, 5, 20):
            tok = int(g.integers(0, 1560))
            x = oracle.rope3d_f32(q, (dpos, tok // 52, tok % 52))
            # the block-scale ratio stays at 448 up to the rotation's rounding
            assert np.abs(x).max() / (6 * s) <= 448 * (1 + 2.0 ** -18)
            codes, scales = oracle.q_for_frame(q, dpos, tok, 52, s)
            rc, rs = oracle.quantize_rows(x, s)
            assert np.array_equal(codes, rc) and np.array_equal(scales, rs)
            assert scales.max() <= 0x7E


def test_fp4_block_form_equals_dequantized_dot():
    g = _rng(7)
    for _ in range(200):
        ca, cb = g.integers(0, 256, 64).astype(np.uint8), g.integers(0, 256, 64).astype(np.uint8)
        sa, sb = g.integers(0, 0x7F, 8).astype(np.uint8), g.integers(0, 0x7F, 8).astype(np.uint8)
        ga, gb = np.float32(np.exp(g.uniform(-20, 5))), np.float32(np.exp(g.uniform(-20, 5)))
        da = oracle.dequant_rows(ca, sa, ga)
        db = oracle.dequant_rows(cb, sb, gb)
        ref = float(np.dot(da, db))
        got = oracle.fp4_dot(ca, sa, ga, cb, sb, gb)
        assert abs(got - ref) <= 1e-13 * max(1e-300, float(np.dot(np.abs(da), np.abs(db))))
    # a hand example: every element code 0x2 (1.0) against code 0x7 (6.0),
    # block scales 1.0 (0x38) and 2.0 (0x40), global scales 1: 128 * 12 = 1536
    one = np.full(64, 0x22, np.uint8)
    six = np.full(64, 0x77, np.uint8)
    assert oracle.fp4_dot(one, np.full(8, 0x38, np.uint8), 1.0, six,
                          np.full(8, 0x40, np.uint8), 1.0) == 1536.0


def _exact_row(g, k_exp):
    """A row that NVFP4 holds exactly under its own per-row scale: in each
    block one pair (6, 0) and the other pairs of magnitude below 6, all times
    448 * 2^k_exp, so s_gq = 2^k_exp and every block scale is 448."""
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4], np.float64)
    x = np.zeros(128)
    for blk in range(8):
        vals = g.choice(mags, 16) * g.choice([-1, 1], 16)
        p = 2 * int(g.integers(0, 8))                            # the pair (6, 0)
        vals[p], vals[p + 1] = 6.0, 0.0
        x[blk * 16:(blk + 1) * 16] = vals
    return (x * 448.0 * 2.0 ** k_exp).astype(np.float32)


def test_fp4_path_equals_current_path_when_q_is_exact():
    g = _rng(11)
    Lq, Lk = 6, 50
    q = np.stack([_exact_row(g, k) for k in g.integers(-6, 3, Lq)])
    assert np.array_equal(_bf16(q), q)
    for r in range(Lq):
        s = oracle.q_row_global_scale(q[r])
        c, sc = oracle.q_for_frame(q[r], 0, 0, 8, s)
        assert np.array_equal(oracle.dequant_rows(c, sc, s), q[r].astype(np.float64))
    # keys at token 0 of the query's own frame index: every rotation trivial
    k = _bf16(g.standard_normal((Lk, 128)))
    v = g.standard_normal((Lk, 128))
    kpos = np.full(Lk, 4, np.int32)
    ktok = np.zeros(Lk, np.int32)
    qpos = np.full(Lq, 4, np.int32)
    qtok = np.zeros(Lq, np.int32)
    rows = np.arange(Lq)
    s_g = oracle.global_scale(oracle.amax(k))
    kc, ks = oracle.quantize_rows(k, s_g)
    kd = oracle.dequant_rows(kc, ks, s_g)
    ref, ref_lse = oracle.attention_rows(q, kd, v, kpos, ktok, qpos, qtok, rows, 8)
    got, lse = oracle.attention_rows_fp4qk(q, kd, v, kpos, qpos, qtok, rows, 8)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_fp4_stream_stores_spatially_rotated_keys():
    wl = kvsynth.WORKLOADS["tiny"]
    a = OracleStream(wl, seed=4, fp4_qk=True)
    x = kvsynth.chunk_qkv(wl, 1, 4)
    new = a.step(k=x["k"], v=x["v"], q=x["q"])
    kf = x["k"].float().numpy()[0]                            # [Lq, H, 128]
    tok = (np.arange(wl.Lq) % wl.T).astype(np.int32)
    for h in range(wl.H):
        kp = oracle.k_spatial_rope_f32(kf[:, h], tok, wl.grid_w)
        assert a.s_g[0, 0, h] == oracle.global_scale(oracle.amax(kp))
        e = a.frame(0, new[0][0])
        codes, scales = oracle.quantize_rows(kp[:wl.T], a.s_g[0, 0, h])
        assert np.array_equal(e["k_codes"][h], codes) and np.array_equal(e["k_scales"][h], scales)
