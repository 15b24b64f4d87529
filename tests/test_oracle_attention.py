"""Pins for the oracle's RoPE and attention (CPU only).

RoPE: invariants that any rotary encoding must satisfy (norm preservation,
identity at position 0, composition of rotations, dependence of q.k on the
position difference only) plus a complex-number restatement of the pair
rotation.  The pairing/frequency convention itself is a reading (adjacent
pairs, base^(-2i/d) per axis); beyond these invariants it is parity unpinned.

Attention: checked against numpy/scipy fp64 softmax(QK^T/sqrt(D))V and
logsumexp on RoPE-rotated inputs, and against closed-form special cases.
"""
import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle

SPLIT = oracle.ROPE_SPLIT


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_rope_preserves_norm_and_identity():
    rng = np.random.default_rng(0)
    for _ in range(50):
        x = _rand(rng, 128)
        pos = rng.integers(0, 60, 3)
        y = oracle.rope3d(x, pos)
        assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-12
    x = _rand(rng, 128)
    assert np.array_equal(oracle.rope3d(x, (0, 0, 0)), x)


def test_rope_composition():
    rng = np.random.default_rng(1)
    x = _rand(rng, 128)
    a, b = np.array([3, 5, 7]), np.array([11, 2, 40])
    y = oracle.rope3d(oracle.rope3d(x, a), b)
    assert np.abs(y - oracle.rope3d(x, a + b)).max() < 1e-12


def test_rope_relative_shift_invariance():
    # (R(p) q) . (R(p') k) depends only on p - p' for every axis
    rng = np.random.default_rng(2)
    q, k = _rand(rng, 128), _rand(rng, 128)
    p, pk = np.array([9, 4, 17]), np.array([2, 21, 3])
    ref = oracle.rope3d(q, p) @ oracle.rope3d(k, pk)
    for c in ([5, 0, 0], [0, 7, 0], [0, 0, 13], [100, 3, 9]):
        c = np.array(c)
        assert abs(oracle.rope3d(q, p + c) @ oracle.rope3d(k, pk + c) - ref) < 1e-10


def test_rope_axis_segments_are_independent():
    # moving along one axis only touches that axis' channel segment
    rng = np.random.default_rng(3)
    x = _rand(rng, 128)
    bounds = np.cumsum((0,) + SPLIT)
    for ax in range(3):
        pos = [0, 0, 0]
        pos[ax] = 5
        y = oracle.rope3d(x, pos)
        changed = np.nonzero(np.abs(y - x) > 0)[0]
        assert changed.min() >= bounds[ax] and changed.max() < bounds[ax + 1]


def test_rope_matches_complex_rotation():
    # pair (x_2i, x_2i+1) as the complex number x_2i + i x_2i+1, times e^(i*phi)
    rng = np.random.default_rng(4)
    x = _rand(rng, 128)
    pos = (6, 13, 29)
    y = oracle.rope3d(x, pos)
    off = 0
    for ax, d in enumerate(SPLIT):
        z = x[off:off + d:2] + 1j * x[off + 1:off + d:2]
        freqs = np.exp(-np.log(oracle.ROPE_BASE) * np.arange(0, d, 2) / d)
        w = z * np.exp(1j * pos[ax] * freqs)
        assert np.abs(y[off:off + d:2] - w.real).max() < 1e-12
        assert np.abs(y[off + 1:off + d:2] - w.imag).max() < 1e-12
        off += d


def _reference_attention(q, k, v, kpos, qpos):
    qr = np.stack([oracle.rope3d(q[i], qpos[i]) for i in range(len(q))])
    kr = np.stack([oracle.rope3d(k[j], kpos[j]) for j in range(len(k))])
    logits = qr @ kr.T / np.sqrt(128.0)
    return softmax(logits, axis=1) @ v, logsumexp(logits, axis=1)


def test_attention_matches_numpy_softmax():
    rng = np.random.default_rng(5)
    grid_w = 6
    Lq, Lk = 9, 53
    q = rng.standard_normal((Lq, 128)).astype(np.float32)
    k, v = rng.standard_normal((Lk, 128)) * 2, rng.standard_normal((Lk, 128))
    kf, kt = rng.integers(0, 5, Lk).astype(np.int32), rng.integers(0, 36, Lk).astype(np.int32)
    qf, qt = np.full(Lq, 5, np.int32), rng.integers(0, 36, Lq).astype(np.int32)
    out, lse = oracle.attention_rows(q, k, v, kf, kt, qf, qt, np.arange(Lq), grid_w)
    kpos = np.stack([kf, kt // grid_w, kt % grid_w], 1)
    qpos = np.stack([qf, qt // grid_w, qt % grid_w], 1)
    ref, ref_lse = _reference_attention(q.astype(np.float64), k, v, kpos, qpos)
    assert np.abs(out - ref).max() < 1e-12
    assert np.abs(lse - ref_lse).max() < 1e-12


def test_attention_row_subset_and_key_permutation():
    rng = np.random.default_rng(6)
    Lq, Lk, grid_w = 7, 40, 8
    q = rng.standard_normal((Lq, 128)).astype(np.float32)
    k, v = rng.standard_normal((Lk, 128)), rng.standard_normal((Lk, 128))
    kf, kt = rng.integers(0, 4, Lk).astype(np.int32), rng.integers(0, 64, Lk).astype(np.int32)
    qf, qt = np.full(Lq, 4, np.int32), np.arange(Lq, dtype=np.int32)
    full, _ = oracle.attention_rows(q, k, v, kf, kt, qf, qt, np.arange(Lq), grid_w)
    rows = np.array([5, 1])
    sub, _ = oracle.attention_rows(q, k, v, kf, kt, qf, qt, rows, grid_w)
    assert np.array_equal(sub, full[rows])
    p = rng.permutation(Lk)
    perm, _ = oracle.attention_rows(q, k[p], v[p], kf[p], kt[p], qf, qt, np.arange(Lq), grid_w)
    assert np.abs(perm - full).max() < 1e-12


def test_attention_special_cases():
    rng = np.random.default_rng(8)
    q = rng.standard_normal((3, 128)).astype(np.float32)
    v1 = rng.standard_normal((1, 128))
    z = np.zeros(1, np.int32)
    out, lse = oracle.attention_rows(q, rng.standard_normal((1, 128)), v1, z, z,
                                     np.zeros(3, np.int32), np.zeros(3, np.int32), np.arange(3), 8)
    assert np.abs(out - v1).max() < 1e-15          # one key: output is its value
    vs = rng.standard_normal((10, 128))
    zk = np.zeros((10, 128))
    z10 = np.zeros(10, np.int32)
    out, lse = oracle.attention_rows(q, zk, vs, z10, z10, np.zeros(3, np.int32),
                                     np.zeros(3, np.int32), np.arange(3), 8)
    assert np.abs(out - vs.mean(0)).max() < 1e-14  # equal logits: plain mean
    assert np.abs(lse - np.log(10.0)).max() < 1e-14
