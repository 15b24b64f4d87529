"""Pins of the sequence-parallel merge oracle (CPU only).

The merge is pinned to the definition of softmax attention computed directly
over all keys (not through the merge formula), to its special cases, and the
oracle stream's per-shard attention to its whole-cache attention."""
import numpy as np
import pytest

import kvsynth
from oracle.merge import lse_merge, shard_tokens
from oracle.stream import OracleStream


def _softmax_attention(s, v):
    """Direct softmax attention of one query: (out [128], log normaliser)."""
    m = s.max()
    e = np.exp(s - m)
    return (e[:, None] * v).sum(0) / e.sum(), m + np.log(e.sum())


@pytest.mark.parametrize("seed", range(5))
@pytest.mark.parametrize("n", [1, 2, 3, 7])
def test_merge_of_a_partition_is_attention_over_all_keys(seed, n):
    rng = np.random.default_rng(seed * 10 + n)
    Lk = 97
    s = rng.normal(0, 3, Lk)
    v = rng.normal(0, 1, (Lk, 128))
    full_o, full_l = _softmax_attention(s, v)
    part = rng.integers(0, n, Lk)
    o_parts, l_parts = [], []
    for j in range(n):
        idx = np.nonzero(part == j)[0]
        if idx.size == 0:
            o_parts.append(np.full(128, np.nan))   # garbage: must carry no weight
            l_parts.append(-np.inf)
        else:
            o, l = _softmax_attention(s[idx], v[idx])
            o_parts.append(o)
            l_parts.append(l)
    o, l = lse_merge(o_parts, [np.float64(x) for x in l_parts])
    np.testing.assert_allclose(o, full_o, rtol=1e-12, atol=1e-12)
    assert abs(l - full_l) < 1e-12


def test_single_part_is_identity():
    rng = np.random.default_rng(3)
    o = rng.normal(size=(5, 128))
    l = rng.normal(size=5)
    mo, ml = lse_merge([o], [l])
    np.testing.assert_array_equal(mo, o)
    np.testing.assert_array_equal(ml, l)


def test_two_equal_parts():
    # the same key set twice: same output, normaliser doubled
    rng = np.random.default_rng(4)
    o = rng.normal(size=(3, 128))
    l = rng.normal(size=3)
    mo, ml = lse_merge([o, o], [l, l])
    np.testing.assert_allclose(mo, o, rtol=1e-14)
    np.testing.assert_allclose(ml, l + np.log(2.0), rtol=1e-14)


def test_weights_follow_the_normalisers():
    # L_1 - L_2 = ln 3: the first part carries 3/4 of the weight
    o1, o2 = np.ones(128), np.zeros(128)
    mo, ml = lse_merge([o1, o2], [np.float64(np.log(3.0)), np.float64(0.0)])
    np.testing.assert_allclose(mo, 0.75, rtol=1e-14)
    assert abs(ml - np.log(4.0)) < 1e-14


def test_no_keys_anywhere():
    mo, ml = lse_merge([np.full(128, np.nan)] * 3, [np.float64(-np.inf)] * 3)
    assert np.all(mo == 0) and ml == -np.inf


def test_shard_tokens():
    assert shard_tokens(1560, 4, 3) == (1170, 1560)
    assert shard_tokens(64, 1, 0) == (0, 64)
    for bad in [(1560, 7, 0), (64, 2, 2), (64, 0, 0)]:
        with pytest.raises(ValueError):
            shard_tokens(*bad)


@pytest.mark.parametrize("count", [2, 4])
def test_sharded_stream_attention_merges_to_the_whole(count):
    wl = kvsynth.WORKLOADS["tiny"]
    ora = OracleStream(wl, seed=1)
    for _ in range(4):
        ora.step()
    rows = np.arange(0, wl.Lq, 7)
    for h in range(wl.H):
        full_o, full_l = ora.attention(0, h, rows)
        parts = [ora.attention(0, h, rows, tokens=shard_tokens(wl.T, count, r)) for r in range(count)]
        o, l = lse_merge([p[0] for p in parts], [p[1] for p in parts])
        np.testing.assert_allclose(o, full_o, rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(l, full_l, rtol=1e-12)
